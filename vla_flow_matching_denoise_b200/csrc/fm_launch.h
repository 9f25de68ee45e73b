// Host-side launch wrappers of the kernels (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "fm_batch.h"
#include "fm_internal.h"

namespace fm {

cudaError_t launch_pack(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                        const uint16_t* const* mats, const int* mat_k, uint8_t* dst,
                        cudaStream_t st);
cudaError_t launch_pack8(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                         const uint8_t* const* mats, const int* mat_k, uint8_t* dst, cudaStream_t st);
cudaError_t launch_pack8_tile(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                              const uint8_t* const* mats, const int* mat_k, uint8_t* dst, cudaStream_t st);
cudaError_t launch_nvfp4_quantize(const uint16_t* w, int rows, int K, unsigned int* amax_scratch, uint8_t* codes,
                                  uint8_t* sb, float* g, cudaStream_t st);
cudaError_t launch_pack_nvfp4(const PackChunk* chunks, int nchunks, const int32_t* rowidx, const uint8_t* codes,
                              const uint8_t* sb, int K, uint8_t* dst, cudaStream_t st);
cudaError_t launch_fp8_quantize(const uint16_t* w, int rows, int K, float* scale, uint8_t* q,
                                cudaStream_t st);
cudaError_t launch_kv_copy(const uint16_t* src, int B, int P, const int* lens, int Hkv, int hd, int S_max,
                           uint16_t* cache, cudaStream_t st);
cudaError_t launch_rope_table(int B, int T, int hd, const int* P, double base, float* tab, cudaStream_t st);
cudaError_t launch_transpose_bf16(const uint16_t* src, int rows, int cols, uint16_t* dst, cudaStream_t st);

size_t time_gemm_smem_bytes(int d);
cudaError_t launch_time(const TimeParams& p, int n_sms, cudaStream_t st);

// Latency-mode denoise megakernel (one request, persistent, clusters of 8).
size_t step_smem_bytes();
cudaError_t step_max_clusters(int* n_clusters);
cudaError_t launch_step(const StepParams& p, cudaStream_t st);

// Batched path (B requests per step, M = B * T rows).
int bgemm_bn(int epi, int N);   // weight tile width the GEMM uses for this epilogue
cudaError_t launch_bgemm(const BGemmParams& p, int epi, int n_sms, cudaStream_t st);
cudaError_t launch_binproj(const BRowParams& p, cudaStream_t st);
cudaError_t launch_rows_to_act128(const uint16_t* src, int M, int Mp, int K, uint16_t* dst, cudaStream_t st);
cudaError_t launch_bresnorm(const BRowParams& p, cudaStream_t st);
cudaError_t launch_browquant(const BQuantParams& p, cudaStream_t st);
cudaError_t launch_boutproj(const BRowParams& p, cudaStream_t st);
cudaError_t launch_battn(const BAttnParams& p, cudaStream_t st);
// tcgen05 attention: every request's keys (P_b + T <= S_max <= 384) in TMEM at once
bool battn_tc_supported(int S_max, int hd);
cudaError_t launch_battn_tc(const BAttnParams& p, cudaStream_t st);

// Sets the text fm_last_error(NULL) returns on this thread.
void set_thread_error(const char* msg);

}  // namespace fm
