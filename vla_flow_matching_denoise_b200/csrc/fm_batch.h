// Parameter structures of the batched (throughput) path's kernels, shared by
// the host engine (fm_api.cu) and fm_batch.cu.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "fm_internal.h"

namespace fm {

// ---------------------------------------------------------------- batched path
// Layout "ACT128": a bf16 activation matrix of Mp rows (Mp a multiple of 128;
// row m = b * T + t for request b, token t) stored as [Mp/128][K/64] blocks of
// 128 rows x 128 bytes (16 KB), 16-byte pieces swizzled by (row & 7): the
// image tcgen05.mma reads for an M = 128 operand.  Packed batched weights:
// [N/BN][K/64] chunks of BN rows x 64 columns in the same swizzled image.
constexpr int kBM = 128;               // rows per batched GEMM tile
constexpr int kBRing = 192 * 1024;     // batched GEMM operand ring

enum BEpi { BE_QKV = 0, BE_RESID = 1, BE_SWIGLU = 2 };

struct BGemmParams {
  // bf16 operands: A is ACT128 [Mp/128][K/64], W packed [N/BN][K/64] chunks of
  // BN x 64.  E4M3 operands (the W8A8 variant): A is ACT8 [Mp/128][K/128], W
  // [N/BN][K/128] chunks of BN x 128 codes; both 128-byte rows, same swizzle.
  const uint8_t* A;
  const uint8_t* W;
  int K, N, M, Mp;           // reduction, output channels, valid rows (B*T), padded rows
  const float* a_scale;      // E4M3 only: [Mp] row scale of A (per token)
  const float* w_scale;      // E4M3 only: [N] scale of the weight row behind each GEMM column
  // BE_RESID: h[m][n] += gate[n] * D[m][n] (fp32 residual, row stride N; one
  // atomic add per element: tiles are disjoint, so no order dependence)
  float* h;
  const float* gate;
  // BE_SWIGLU: tile j holds gate rows 128j.. then up rows 128j..; u = SiLU(g) up
  uint16_t* u_act;           // ACT128 [Mp/128][F/64]
  int F;
  // BE_QKV: RoPE on q, k; q -> qbuf [B][Hkv][q_rows][hd]; k, v -> cache rows
  // P_b + t of request b = m / T, t = m % T.  The prefix cache builder uses the
  // same epilogue with no q heads (Hq = 0), T = the prefix length, P_dev null
  // (rows start at 0) and one RoPE table shared by all requests.
  uint16_t* qbuf;
  uint16_t* kc;              // this layer's K cache [B_cap][Hkv][S_max][hd]
  uint16_t* vc;
  const float* rope;         // (cos, sin) rows [b * rope_stride_b + t][hd/2]
  int rope_stride_b;         // T for the chunk (per-request positions), 0 for the prefix
  const int* P_dev;          // [B_cap] prefix length per request, or null (offset 0)
  int T, Hq, Hkv, hd, S_max, q_rows;
  uint32_t* err;
  long long spin_budget;
};

struct BRowParams {          // in-proj, AdaRMSNorm, out-proj + Euler (row kernels)
  int M, T, A, d;
  float eps, dt;
  const float* x;            // [M][A] (in-proj input)
  float* x_out;              // [M][A] updated in place by out-proj (x += dt v), or null
  float* v_out;              // [M][A] velocity
  const uint16_t* w_in_t;    // [A][d]: the in-projection's weights, transposed
  const uint16_t* w_out;     // [A][d]
  const float* out_bias;     // [A] or null
  float* h;                  // [Mp][d] fp32 residual
  const float* s;            // norm scale and shift [d]
  const float* b;
  uint16_t* z;               // ACT128 [Mp/128][d/64] (bf16), or ACT8 codes when zs is set
  float* zs;                 // non-null: z gets E4M3 codes [Mp/128][d/128] and zs[m] their row scale
};

// Per-token E4M3 of a bf16 ACT128 matrix [M][K] into ACT8 codes and row scales.
struct BQuantParams {
  const uint16_t* src;       // ACT128 [Mp/128][K/64]
  uint8_t* dst;              // ACT8 [Mp/128][K/128]
  float* scale;              // [Mp]
  int M, K;
};

struct BAttnParams {
  // tensor-core kernel: 4-D views (64 elements, hd/64 halves, rows, segments)
  // of the q buffer (segment b Hkv + g) and of the K/V caches (segment
  // (l B_cap + b) Hkv + g), box (64, 1, 128, 1): one TMA copy moves 128 half rows
  CUtensorMap tm_q, tm_k, tm_v;
  int seg_base;              // l B_cap Hkv: first cache segment of this layer
  const uint16_t* qbuf;      // [B][Hkv][q_rows][hd]
  const uint16_t* kc;        // this layer's cache [B_cap][Hkv][S_max][hd]
  const uint16_t* vc;
  uint16_t* o_act;           // ACT128 [Mp/128][Hq*hd/64]
  const int* P_dev;          // [B_cap] prefix length per request
  int B, T, Hq, Hkv, hd, S_max, q_rows, qblocks;
  uint32_t* err;
  long long spin_budget;
};

}  // namespace fm
