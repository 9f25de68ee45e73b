// Set-up kernels (run at fm_expert_create / fm_set_prefix, not in the loop):
//  * weight packing into the swizzled, per-CTA-ordered arena (bf16 or E4M3);
//  * per-row absmax scales and E4M3 quantisation of the per-layer linears;
//  * prefix K/V copy into the swizzled KV cache;
//  * the RoPE cos/sin table for the chunk positions P .. P+T-1.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "fm_internal.h"
#include "fm_launch.h"

namespace fm {

// Copies 16-byte pieces of source rows into the swizzled chunk image.
__global__ void pack_kernel(const PackChunk* __restrict__ chunks, const int32_t* __restrict__ rowidx,
                            const uint16_t* const* __restrict__ mats, const int* __restrict__ mat_k,
                            uint8_t* __restrict__ dst) {
  const PackChunk ch = chunks[blockIdx.x];
  const uint16_t* src = mats[ch.mat];
  const int K = mat_k[ch.mat];
  const int pieces = ch.nrows * 8;
  for (int p = threadIdx.x; p < pieces; p += blockDim.x) {
    const int row = p >> 3, c = p & 7;
    const int sr = rowidx[ch.rowidx_off + row];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (sr >= 0) v = *reinterpret_cast<const uint4*>(src + (size_t)sr * K + (size_t)ch.kb * 64 + c * 8);
    *reinterpret_cast<uint4*>(dst + ch.dst_off + (size_t)row * 128 + ((c ^ (row & 7)) << 4)) = v;
  }
}

// Copies 16-byte pieces of E4M3 code rows (one byte per weight) into a chunk
// of R rows x 64 codes, row-major, unswizzled.
__global__ void pack8_kernel(const PackChunk* __restrict__ chunks, const int32_t* __restrict__ rowidx,
                             const uint8_t* const* __restrict__ mats, const int* __restrict__ mat_k,
                             uint8_t* __restrict__ dst) {
  const PackChunk ch = chunks[blockIdx.x];
  if (ch.fmt != 1) return;   // not an E4M3 chunk (NVFP4 chunks have their own packer)
  const uint8_t* src = mats[ch.mat];
  const int K = mat_k[ch.mat];
  const int pieces = ch.nrows * 4;
  for (int p = threadIdx.x; p < pieces; p += blockDim.x) {
    const int row = p >> 2, c = p & 3;
    const int sr = rowidx[ch.rowidx_off + row];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (sr >= 0) v = *reinterpret_cast<const uint4*>(src + (size_t)sr * K + (size_t)ch.kb * 64 + c * 16);
    *reinterpret_cast<uint4*>(dst + ch.dst_off + (size_t)row * 64 + c * 16) = v;
  }
}

// Copies 16-byte pieces of E4M3 code rows into a tensor-core tile chunk of
// R rows x 128 codes (column block ch.kb of 128), pieces swizzled by (row & 7)
// as in the bf16 chunks: the batched W8A8 GEMM's weight layout.
__global__ void pack8_tile_kernel(const PackChunk* __restrict__ chunks, const int32_t* __restrict__ rowidx,
                                  const uint8_t* const* __restrict__ mats, const int* __restrict__ mat_k,
                                  uint8_t* __restrict__ dst) {
  const PackChunk ch = chunks[blockIdx.x];
  const uint8_t* src = mats[ch.mat];
  const int K = mat_k[ch.mat];
  const int pieces = ch.nrows * 8;
  for (int p = threadIdx.x; p < pieces; p += blockDim.x) {
    const int row = p >> 3, c = p & 7;
    const int sr = rowidx[ch.rowidx_off + row];
    uint4 v = make_uint4(0, 0, 0, 0);
    if (sr >= 0) v = *reinterpret_cast<const uint4*>(src + (size_t)sr * K + (size_t)ch.kb * 128 + c * 16);
    *reinterpret_cast<uint4*>(dst + ch.dst_off + (size_t)row * 128 + ((c ^ (row & 7)) << 4)) = v;
  }
}

// Per-row absmax / 448 of a bf16 matrix [rows, K] (R8: s = absmax / 448, 1 for
// an all-zero row).  One warp per row.
__global__ void fp8_row_scale_kernel(const uint16_t* __restrict__ w, int rows, int K,
                                     float* __restrict__ scale) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  float m = 0.f;
  for (int k = lane; k < K; k += 32) {
    const float x = __uint_as_float((uint32_t)w[(size_t)warp * K + k] << 16);
    m = fmaxf(m, fabsf(x));
  }
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) scale[warp] = m > 0.f ? __fdiv_rn(m, 448.0f) : 1.0f;
}

// E4M3 codes of w / s (true fp32 division, nearest-even, saturating finite).
__global__ void fp8_quantize_kernel(const uint16_t* __restrict__ w, const float* __restrict__ scale,
                                    int rows, int K, uint8_t* __restrict__ q) {
  const size_t n = (size_t)rows * K;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x) {
    const float x = __uint_as_float((uint32_t)w[i] << 16);
    const float r = __fdiv_rn(x, scale[i / K]);
    q[i] = (uint8_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
  }
}

// Largest |w| of a bf16 tensor, as the bits of a non-negative float (their
// integer order is the float order, so the max is order-independent).
__global__ void absmax_kernel(const uint16_t* __restrict__ w, size_t n, unsigned int* __restrict__ out) {
  float m = 0.f;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(__uint_as_float((uint32_t)w[i] << 16)));
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(out, __float_as_uint(m));
}

// Nearest E2M1 magnitude code of |r| (r finite, fp32), ties to the even code,
// saturating at 6: the E2M1 grid is 0, 0.5, 1, 1.5, 2, 3, 4, 6 and every
// midpoint is exact in fp32.
__device__ __forceinline__ uint32_t e2m1_code(float r) {
  const float a = fabsf(r);
  uint32_t m;
  if (a <= 0.25f) m = 0;
  else if (a < 0.75f) m = 1;
  else if (a <= 1.25f) m = 2;
  else if (a < 1.75f) m = 3;
  else if (a <= 2.5f) m = 4;
  else if (a < 3.5f) m = 5;
  else if (a <= 5.0f) m = 6;
  else m = 7;
  return (m != 0 && r < 0.f) ? (m | 8u) : m;
}

// R10 NVFP4 of a bf16 tensor [rows, K]: g = amax / (6 * 448); per row and
// 16-column block s_b = E4M3(amax_b / (6 g)); codes = E2M1(w / (s_b g)).
// One warp per (row, block); codes one per byte [rows][K], scales [rows][K/16].
__global__ void nvfp4_quantize_kernel(const uint16_t* __restrict__ w, int rows, int K,
                                      const unsigned int* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                                      uint8_t* __restrict__ sb, float* __restrict__ g_out) {
  const float amax = __uint_as_float(*amax_bits);
  const float g = amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
  const int nb = K / 16;
  const size_t total = (size_t)rows * nb;
  const int lane = threadIdx.x & 31;
  for (size_t blk = (blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5; blk < total;
       blk += ((size_t)gridDim.x * blockDim.x) >> 5) {
    const size_t base = blk * 16;
    const float x = lane < 16 ? __uint_as_float((uint32_t)w[base + lane] << 16) : 0.f;
    float m = fabsf(x);
    for (int o = 8; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const uint8_t sc = (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(m, __fmul_rn(6.0f, g)), __NV_SATFINITE, __NV_E4M3);
    const __half_raw hr = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)sc, __NV_E4M3);
    const float sv = __half2float(*reinterpret_cast<const __half*>(&hr));
    const float denom = __fmul_rn(sv, g);
    if (lane < 16) codes[base + lane] = (uint8_t)(denom > 0.f ? e2m1_code(__fdiv_rn(x, denom)) : 0u);
    if (lane == 0) sb[blk] = sc;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *g_out = g;
}

// NVFP4 chunks of the step kernel: R rows x 64 columns = R x 32 bytes of codes
// (two per byte, first element in the low nibble), then R x 4 E4M3 block scales.
__global__ void pack_nvfp4_kernel(const PackChunk* __restrict__ chunks, const int32_t* __restrict__ rowidx,
                                  const uint8_t* __restrict__ codes, const uint8_t* __restrict__ sb, int K,
                                  uint8_t* __restrict__ dst) {
  const PackChunk ch = chunks[blockIdx.x];
  if (ch.fmt != 2) return;   // only NVFP4 chunks
  const int R = ch.nrows;
  for (int q = threadIdx.x; q < R; q += blockDim.x) {
    const int sr = rowidx[ch.rowidx_off + q];
    uint8_t* crow = dst + ch.dst_off + (size_t)q * 32;
    uint8_t* srow = dst + ch.dst_off + (size_t)R * 32 + (size_t)q * 4;
    for (int i = 0; i < 32; ++i) {
      uint8_t v = 0;
      if (sr >= 0) {
        const uint8_t* c = codes + (size_t)sr * K + (size_t)ch.kb * 64 + 2 * i;
        v = (uint8_t)(c[0] | (c[1] << 4));
      }
      crow[i] = v;
    }
    for (int b = 0; b < 4; ++b) srow[b] = sr >= 0 ? sb[(size_t)sr * (K / 16) + (size_t)ch.kb * 4 + b] : 0;
  }
}

// Prefix K or V of one layer: src [B, P_pad, H_kv, hd] -> cache
// [B_cap][H_kv][S_max][hd] with 16-byte pieces swizzled by (row & 7).  Only
// the first lens[b] rows of request b are copied (the rest is padding).
__global__ void kv_copy_kernel(const uint16_t* __restrict__ src, int B, int P, const int* __restrict__ lens,
                               int Hkv, int hd, int S_max, uint16_t* __restrict__ cache) {
  const int pieces = hd / 8;
  const size_t total = (size_t)B * P * Hkv * pieces;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total;
       i += (size_t)gridDim.x * blockDim.x) {
    const int c = (int)(i % pieces);
    size_t r = i / pieces;
    const int g = (int)(r % Hkv); r /= Hkv;
    const int s = (int)(r % P);
    const int b = (int)(r / P);
    if (s >= lens[b]) continue;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (((size_t)b * P + s) * Hkv + g) * hd + c * 8);
    uint16_t* row = cache + (((size_t)b * Hkv + g) * S_max + s) * hd;
    *reinterpret_cast<uint4*>(row + ((c ^ (s & 7)) << 3)) = v;
  }
}

// cos / sin of pos * base^(-2i/hd) for pos = P_b + t of every request b, in
// double, stored fp32: tab [B][T][hd/2][2].
__global__ void rope_table_kernel(int B, int T, int hd, const int* __restrict__ P, double base,
                                  float* __restrict__ tab) {
  const int half = hd / 2;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * T * half) return;
  const int b = i / (T * half), t = (i / half) % T, j = i % half;
  const double theta = pow(base, -2.0 * j / hd);
  const double ang = (double)(P[b] + t) * theta;
  tab[2 * i] = (float)cos(ang);
  tab[2 * i + 1] = (float)sin(ang);
}

// dst[c][r] = src[r][c] for a bf16 matrix [rows][cols].
__global__ void transpose_bf16_kernel(const uint16_t* __restrict__ src, int rows, int cols,
                                      uint16_t* __restrict__ dst) {
  const size_t n = (size_t)rows * cols;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const size_t r = i / cols, c = i % cols;
    dst[c * rows + r] = src[i];
  }
}

cudaError_t launch_transpose_bf16(const uint16_t* src, int rows, int cols, uint16_t* dst, cudaStream_t st) {
  transpose_bf16_kernel<<<256, 256, 0, st>>>(src, rows, cols, dst);
  return cudaGetLastError();
}

cudaError_t launch_pack(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                        const uint16_t* const* mats, const int* mat_k, uint8_t* dst,
                        cudaStream_t st) {
  if (nchunks == 0) return cudaSuccess;
  pack_kernel<<<nchunks, 256, 0, st>>>(chunks, rowidx, mats, mat_k, dst);
  return cudaGetLastError();
}

cudaError_t launch_pack8(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                         const uint8_t* const* mats, const int* mat_k, uint8_t* dst, cudaStream_t st) {
  if (nchunks == 0) return cudaSuccess;
  pack8_kernel<<<nchunks, 256, 0, st>>>(chunks, rowidx, mats, mat_k, dst);
  return cudaGetLastError();
}

cudaError_t launch_pack8_tile(const PackChunk* chunks, int nchunks, const int32_t* rowidx,
                              const uint8_t* const* mats, const int* mat_k, uint8_t* dst, cudaStream_t st) {
  if (nchunks == 0) return cudaSuccess;
  pack8_tile_kernel<<<nchunks, 256, 0, st>>>(chunks, rowidx, mats, mat_k, dst);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_quantize(const uint16_t* w, int rows, int K, unsigned int* amax_scratch, uint8_t* codes,
                                  uint8_t* sb, float* g, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(amax_scratch, 0, 4, st);
  if (e != cudaSuccess) return e;
  absmax_kernel<<<512, 256, 0, st>>>(w, (size_t)rows * K, amax_scratch);
  nvfp4_quantize_kernel<<<1024, 256, 0, st>>>(w, rows, K, amax_scratch, codes, sb, g);
  return cudaGetLastError();
}

cudaError_t launch_pack_nvfp4(const PackChunk* chunks, int nchunks, const int32_t* rowidx, const uint8_t* codes,
                              const uint8_t* sb, int K, uint8_t* dst, cudaStream_t st) {
  if (nchunks == 0) return cudaSuccess;
  pack_nvfp4_kernel<<<nchunks, 128, 0, st>>>(chunks, rowidx, codes, sb, K, dst);
  return cudaGetLastError();
}

cudaError_t launch_fp8_quantize(const uint16_t* w, int rows, int K, float* scale, uint8_t* q,
                                cudaStream_t st) {
  fp8_row_scale_kernel<<<(rows * 32 + 255) / 256, 256, 0, st>>>(w, rows, K, scale);
  fp8_quantize_kernel<<<1024, 256, 0, st>>>(w, scale, rows, K, q);
  return cudaGetLastError();
}

cudaError_t launch_kv_copy(const uint16_t* src, int B, int P, const int* lens, int Hkv, int hd, int S_max,
                           uint16_t* cache, cudaStream_t st) {
  if ((size_t)B * P == 0) return cudaSuccess;
  kv_copy_kernel<<<512, 256, 0, st>>>(src, B, P, lens, Hkv, hd, S_max, cache);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(int B, int T, int hd, const int* P, double base, float* tab, cudaStream_t st) {
  const int n = B * T * hd / 2;
  rope_table_kernel<<<(n + 127) / 128, 128, 0, st>>>(B, T, hd, P, base, tab);
  return cudaGetLastError();
}

}  // namespace fm
