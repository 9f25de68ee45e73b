// Batched (throughput) path of the denoise loop: B requests advance through
// each Euler step together, so every per-layer linear sees M = B * T token
// rows (3200 at B = 64) and is a real tensor-core GEMM rather than a weight
// stream.  The request-independence of the loop ("LingBot-VLA v2 Examples",
// Configuration / CUDA Graph: each request has its own prefix KV cache and a
// fixed-shape denoise graph) lets the batch share each weight tile.
//
// One Euler step is a chain of launches (captured in one CUDA graph per
// (B, n) by the host):
//   in-proj -> AdaRMSNorm -> L x (QKV GEMM + RoPE -> GQA attention -> o_proj
//   GEMM adding its gated branch into h -> AdaRMSNorm -> gate_up GEMM + SwiGLU
//   -> down GEMM adding its gated branch into h -> AdaRMSNorm, except after
//   the last layer) -> final AdaRMSNorm + out-proj + Euler.
//
// GEMM (bgemm_kernel): persistent, one CTA per SM.  Warp 0 streams the 16 KB
// A block and the BN x 64 weight chunk of every k-block into a 192 KB ring by
// bulk copy; warp 1 issues tcgen05.mma (M = 128, N = BN, K = 16) into one of
// two TMEM accumulators; warps 2-5 drain the other accumulator through the
// fused epilogue (RoPE + cache scatter, gated residual, or SwiGLU), so the
// epilogue of tile i overlaps the main loop of tile i + 1.  Tiles are ordered
// m-fastest, so the CTAs in flight share each weight chunk through L2.
//
// W8A8 variant: the same kernels with E4M3 operands.  The inputs of the four
// per-layer linears are quantised per token (s = amax_row / 448): the norm
// kernels emit the codes of z directly, a row-quantiser pass follows attention
// (o) and the gate_up GEMM (u).  The GEMM streams 128-byte rows of codes
// (K = 128 per k-block), issues tcgen05.mma kind::f8f6f4 (K = 32 each), and
// the epilogue scales D by s_a[m] s_w[n] before the fused work.
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>
#include <utility>

#include "fm_batch.h"
#include "fm_internal.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {

constexpr int kBEpiWarps = 4;                        // warps 2 .. 5
constexpr int kBThreads = 64 + 32 * kBEpiWarps;

template <int BN>
struct BCfg {
  static constexpr int kA = kBM * 128;          // A block bytes (128 rows x 64 bf16)
  static constexpr int kW = BN * 128;           // weight chunk bytes
  static constexpr int kStage = kA + kW;
  static constexpr int kStages = kBRing / kStage;
  static constexpr size_t kColF = (size_t)kBEpiWarps * BN * 4;   // per-column epilogue factors, per warp
  static constexpr size_t kSmem = 1024 + (size_t)kStages * kStage + 256 + kColF;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Element offset of (row m, column c) in an ACT128 matrix with K columns.
__device__ __forceinline__ size_t act128_off(int m, int c, int K) {
  return ((size_t)(m >> 7) * (K >> 6) + (c >> 6)) * (kBM * 64) + (size_t)(m & 127) * 64 +
         ((((c & 63) >> 3) ^ (m & 7)) << 3) + (c & 7);
}

// Byte offset of (row m, column c) in an ACT8 matrix (E4M3 codes) with K
// columns: blocks of 128 rows x 128 codes, 16-byte pieces swizzled by (m & 7).
__device__ __forceinline__ size_t act8_off(int m, int c, int K) {
  return ((size_t)(m >> 7) * (K >> 7) + (c >> 7)) * (kBM * 128) + (size_t)(m & 127) * 128 +
         ((((c & 127) >> 4) ^ (m & 7)) << 4) + (c & 15);
}

__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// R11 per-token factors of a row with largest magnitude `amax`: the
// dequantisation scale s = amax / 448 and the quantisation factor
// r = 448 / amax (both 1 for a zero row); codes = E4M3(y r).
__device__ __forceinline__ float act_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f; }
__device__ __forceinline__ float act_rcp(float amax) { return amax > 0.f ? __fdiv_rn(448.0f, amax) : 1.0f; }

// E4M3 codes of four values times r, packed little-end first.
__device__ __forceinline__ uint32_t e4m3x4_of(float a, float b, float c, float d, float r) {
  return f32x2_to_e4m3x2(__fmul_rn(a, r), __fmul_rn(b, r)) | (f32x2_to_e4m3x2(__fmul_rn(c, r), __fmul_rn(d, r)) << 16);
}

// Multiplies v[0..15] by sa * sw[0 .. 15] (E4M3 GEMM dequantisation; sw in
// shared memory, the same address for every lane).
__device__ __forceinline__ void dequant16(float (&v)[16], float sa, const float* sw) {
  const float4* w4 = reinterpret_cast<const float4*>(sw);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 w = w4[q];
    v[4 * q] *= sa * w.x;
    v[4 * q + 1] *= sa * w.y;
    v[4 * q + 2] *= sa * w.z;
    v[4 * q + 3] *= sa * w.w;
  }
}

// ------------------------------------------------------------------ epilogues
// Thread = one accumulator row (TMEM lane); `ta` is the TMEM address of column
// 0 of this tile for the thread's lane quarter.

// Gated residual: h[m][n] += gate[n] * D[m][n], one vector atomic add per 4
// elements (no read back into the epilogue; the row kernel that follows
// normalises h).
// `cs`: this tile's column factors in shared memory (gate[n] s_w[n]).
template <int BN, bool F8>
__device__ __forceinline__ void epi_resid(const BGemmParams& p, uint32_t ta, int m, bool valid, int nt,
                                          const float* cs, float sa) {
#pragma unroll 1
  for (int cb = 0; cb < BN / 16; ++cb) {
    float v[16];
    tmem_ld16(ta + cb * 16, v);
    tmem_ld_wait();
    if (!valid) continue;
    const int n0 = nt * BN + cb * 16;
    if (F8) {
#pragma unroll
      for (int i = 0; i < 16; ++i) v[i] *= sa;
    }
    float* hp = p.h + (size_t)m * p.N + n0;
    const float4* gp = reinterpret_cast<const float4*>(cs + cb * 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 g = gp[q];
      red_add_v4(hp + 4 * q, g.x * v[4 * q], g.y * v[4 * q + 1], g.z * v[4 * q + 2], g.w * v[4 * q + 3]);
    }
  }
}

template <int BN, bool F8>
__device__ __forceinline__ void epi_swiglu(const BGemmParams& p, uint32_t ta, int m, bool valid, int nt,
                                           const float* cs, float sa) {
  constexpr int HALF = BN / 2;
#pragma unroll 1
  for (int j = 0; j < HALF / 16; ++j) {
    float g[16], u[16];
    tmem_ld16(ta + j * 16, g);
    tmem_ld16(ta + HALF + j * 16, u);
    tmem_ld_wait();
    if (!valid) continue;
    if (F8) {
      dequant16(g, sa, cs + j * 16);
      dequant16(u, sa, cs + HALF + j * 16);
    }
    const int uc = nt * HALF + j * 16;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) pk[i] = pack2_bf16(silu(g[2 * i]) * u[2 * i], silu(g[2 * i + 1]) * u[2 * i + 1]);
    *reinterpret_cast<uint4*>(p.u_act + act128_off(m, uc, p.F)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    *reinterpret_cast<uint4*>(p.u_act + act128_off(m, uc + 8, p.F)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  }
}

// 16 consecutive elements e0 .. e0 + 15 of a row of hd values stored with
// 16-byte pieces swizzled by (row & 7).
__device__ __forceinline__ void store_row16(uint16_t* rowp, int row, int e0, const float (&y)[16]) {
  uint32_t pk[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) pk[i] = pack2_bf16(y[2 * i], y[2 * i + 1]);
  const int pc = e0 >> 3;
  *reinterpret_cast<uint4*>(rowp + (((pc) ^ (row & 7)) << 3)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  *reinterpret_cast<uint4*>(rowp + (((pc + 1) ^ (row & 7)) << 3)) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
}

template <int BN, bool F8>
__device__ __forceinline__ void epi_qkv(const BGemmParams& p, uint32_t ta, int m, bool valid, int nt,
                                        const float* cs, float sa) {
  const int hd = p.hd, half = hd / 2;
  const int qn = p.Hq * hd, kn = p.Hkv * hd, G = p.Hq / p.Hkv;
  const int b = valid ? m / p.T : 0, t = valid ? m % p.T : 0;
  // chunk: rows and RoPE positions follow this request's prefix length
  const int P = p.P_dev != nullptr ? p.P_dev[b] : 0;
  const float4* rope4 = reinterpret_cast<const float4*>(reinterpret_cast<const float2*>(p.rope) +
                                                        ((size_t)b * p.rope_stride_b + t) * half);
  const int nh = BN / hd;
  auto dst = [&](int h, int& row) -> uint16_t* {
    const int col0 = nt * BN + h * hd;
    const int kind = col0 < qn ? 0 : col0 < qn + kn ? 1 : 2;
    const int head = (kind == 0 ? col0 : kind == 1 ? col0 - qn : col0 - qn - kn) / hd;
    if (kind == 0) {   // (only when Hq > 0)
      row = (head % G) * p.T + t;
      return p.qbuf + (((size_t)b * p.Hkv + head / G) * p.q_rows + row) * hd;
    }
    row = P + t;
    return (kind == 1 ? p.kc : p.vc) + (((size_t)b * p.Hkv + head) * p.S_max + row) * hd;
  };
  auto rotated = [&](int h) { return nt * BN + h * hd < qn + kn; };   // q and k heads take RoPE
  // The tile's q/k heads share this row's (cos, sin) table: each 16-frequency
  // group is loaded once for all of them, one group ahead of its use, so no
  // L2 round trip sits between a TMEM read and its stores.
  float4 rc[8], rn[8];
  if (valid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) rc[i] = rope4[i];
  }
#pragma unroll 1
  for (int c = 0; c < half; c += 16) {
    if (valid && c + 16 < half) {
#pragma unroll
      for (int i = 0; i < 8; ++i) rn[i] = rope4[(c + 16) / 2 + i];
    }
#pragma unroll 1
    for (int h = 0; h < nh; ++h) {
      if (!rotated(h)) continue;
      const int ho = h * hd;
      float lo[16], hi[16];
      tmem_ld16(ta + ho + c, lo);
      tmem_ld16(ta + ho + half + c, hi);
      tmem_ld_wait();
      if (!valid) continue;
      if (F8) {
        dequant16(lo, sa, cs + ho + c);
        dequant16(hi, sa, cs + ho + half + c);
      }
      float ol[16], oh[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 r = rc[i];
        ol[2 * i] = lo[2 * i] * r.x - hi[2 * i] * r.y;
        oh[2 * i] = hi[2 * i] * r.x + lo[2 * i] * r.y;
        ol[2 * i + 1] = lo[2 * i + 1] * r.z - hi[2 * i + 1] * r.w;
        oh[2 * i + 1] = hi[2 * i + 1] * r.z + lo[2 * i + 1] * r.w;
      }
      int row;
      uint16_t* rowp = dst(h, row);
      store_row16(rowp, row, c, ol);
      store_row16(rowp, row, half + c, oh);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) rc[i] = rn[i];
  }
  // v heads: no rotation
#pragma unroll 1
  for (int h = 0; h < nh; ++h) {
    if (rotated(h)) continue;
    const int ho = h * hd;
    int row;
    uint16_t* rowp = dst(h, row);
#pragma unroll 1
    for (int c = 0; c < hd; c += 16) {
      float v[16];
      tmem_ld16(ta + ho + c, v);
      tmem_ld_wait();
      if (!valid) continue;
      if (F8) dequant16(v, sa, cs + ho + c);
      store_row16(rowp, row, c, v);
    }
  }
}

// ------------------------------------------------------------------ GEMM
template <int BN, int EPI, bool F8>
__global__ void __launch_bounds__(kBThreads, 1) bgemm_kernel(const __grid_constant__ BGemmParams p) {
  using C = BCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = align1024(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)C::kStages * C::kStage);
  uint64_t* full = bars;                   // [kStages]
  uint64_t* empty = bars + C::kStages;     // [kStages]
  uint64_t* tfull = empty + C::kStages;    // [2]
  uint64_t* tempty = tfull + 2;            // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  float* colf = reinterpret_cast<float*>(ring + (size_t)C::kStages * C::kStage + 256);   // [4 warps][BN]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = F8 ? p.K / 128 : p.K / 64;   // k-blocks of 128-byte rows
  const int MT = p.Mp / kBM, NT = p.N / BN;
  const int ntiles = MT * NT;   // m-tile fastest
  const long long budget = p.spin_budget;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), kBEpiWarps);
    }
    mbar_init(smem_u32(drain), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();   // A and W are both re-read by other CTAs
      // The weights do not depend on the previous kernel: the first stages'
      // weight chunks are requested before waiting for it.
      int npre = 0;
      if ((int)blockIdx.x < ntiles) {
        npre = nkb < C::kStages ? nkb : C::kStages;
        const uint8_t* w0 = p.W + (size_t)((int)blockIdx.x / MT) * nkb * C::kW;
        for (int j = 0; j < npre; ++j) {
          mbar_expect_tx(smem_u32(&full[j]), C::kW);
          bulk_g2s(smem_u32(ring + (size_t)j * C::kStage + C::kA), w0 + (size_t)j * C::kW, C::kW,
                   smem_u32(&full[j]), pol);
        }
      }
      grid_dep_wait();
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x) {
        const int mt = tile % MT, nt = tile / MT;
        const uint8_t* a_src = p.A + (size_t)mt * nkb * C::kA;
        const uint8_t* w_src = p.W + (size_t)nt * nkb * C::kW;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const uint32_t s = it % C::kStages, ph = (it / C::kStages) & 1;
          if (it >= (uint32_t)C::kStages && !mbar_wait(smem_u32(&empty[s]), ph ^ 1, budget)) {
            atomicOr(p.err, 0x100u);
            ok = false;
            break;
          }
          uint8_t* dst = ring + (size_t)s * C::kStage;
          if ((int)it < npre) {
            mbar_arrive_expect_tx(smem_u32(&full[s]), C::kA);
            bulk_g2s(smem_u32(dst), a_src + (size_t)kb * C::kA, C::kA, smem_u32(&full[s]), pol);
          } else {
            mbar_arrive_expect_tx(smem_u32(&full[s]), C::kStage);
            bulk_g2s(smem_u32(dst), a_src + (size_t)kb * C::kA, C::kA, smem_u32(&full[s]), pol);
            bulk_g2s(smem_u32(dst + C::kA), w_src + (size_t)kb * C::kW, C::kW, smem_u32(&full[s]), pol);
          }
        }
      }
      // every issued copy must land before the CTA may exit
      for (uint32_t j = (it > (uint32_t)C::kStages ? it - C::kStages : 0); j < it; ++j)
        mbar_wait(smem_u32(&full[j % C::kStages]), (j / C::kStages) & 1, budget);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = F8 ? idesc_e4m3(kBM, BN) : idesc_bf16(kBM, BN);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++local) {
        const uint32_t acc = local & 1;
        if (local >= 2 && !mbar_wait(smem_u32(&tempty[acc]), ((local >> 1) - 1) & 1, budget)) {
          atomicOr(p.err, 0x200u);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const uint32_t s = it % C::kStages, ph = (it / C::kStages) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, budget)) {
            atomicOr(p.err, 0x400u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + (size_t)s * C::kStage);
          const uint32_t b_base = a_base + C::kA;
          // four MMAs per 128-byte row: K = 16 bf16 or K = 32 E4M3 each
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            if (F8)
              mma_e4m3(d_tmem, desc_sw128(a_base + k16 * 32), desc_sw128(b_base + k16 * 32), idesc,
                       (kb | k16) != 0);
            else
              mma_bf16(d_tmem, desc_sw128(a_base + k16 * 32), desc_sw128(b_base + k16 * 32), idesc,
                       (kb | k16) != 0);
          }
          mma_commit(smem_u32(&empty[s]));
        }
        if (ok) mma_commit(smem_u32(&tfull[acc]));
      }
      // all issued MMAs must complete before TMEM is released
      mma_commit(smem_u32(drain));
      mbar_wait(smem_u32(drain), 0, budget);
    }
  } else {
    grid_dep_wait();                             // outputs and epilogue operands follow the previous kernel
    const int q4 = warp & 3;                     // TMEM lane quarter this warp may read
    const int row = 32 * q4 + lane;
    // per-column factors, one copy per warp (no cross-warp barrier): gate *
    // s_w (residual), s_w (E4M3 gate_up / QKV)
    constexpr bool kColFactors = EPI == BE_RESID || F8;
    float* cs = colf + (warp - 2) * BN;
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
      const uint32_t acc = local & 1;
      const int mt = tile % MT, nt = tile / MT;
      const int m = mt * kBM + row;
      const bool valid = m < p.M;
      // operands that do not depend on the accumulator are read while the
      // MMAs of this tile still run (the warp finished reading the previous
      // tile's factors before its last __syncwarp)
      if (kColFactors) {
        for (int i = lane; i < BN; i += 32) {
          const int n = nt * BN + i;
          const float w = F8 ? p.w_scale[n] : 1.f;
          cs[i] = EPI == BE_RESID ? p.gate[n] * w : w;
        }
        __syncwarp();
      }
      const float sa = (F8 && valid) ? p.a_scale[m] : 1.f;
      if (!mbar_wait(smem_u32(&tfull[acc]), (local >> 1) & 1, budget)) {
        atomicOr(p.err, 0x800u);
        break;
      }
      tc_fence_after();
      const uint32_t ta = tmem + ((uint32_t)(32 * q4) << 16) + acc * BN;
      if (EPI == BE_RESID) epi_resid<BN, F8>(p, ta, m, valid, nt, cs, sa);
      else if (EPI == BE_SWIGLU) epi_swiglu<BN, F8>(p, ta, m, valid, nt, cs, sa);
      else epi_qkv<BN, F8>(p, ta, m, valid, nt, cs, sa);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

// ------------------------------------------------------------------ row kernels
// In-proj: h = x W_in^T (fp32) for 16 rows x 256 columns per CTA, grid
// (rows / 16, d / 256); thread t computes column 256 blockIdx.y + t for the 16
// rows.  The weights are read transposed (w_in_t [A][d]), so a warp's loads
// for one input are 64 contiguous bytes, four inputs in flight at a time.
// Layer 0's AdaRMSNorm follows in the norm kernel.
constexpr int kRowsIn = 16;
__global__ void __launch_bounds__(256) binproj_kernel(const __grid_constant__ BRowParams p) {
  __shared__ float xs[kRowsIn][128];
  grid_dep_launch();
  grid_dep_wait();
  const int m0 = blockIdx.x * kRowsIn;
  const int tid = threadIdx.x, A = p.A, d = p.d;
  const int n = blockIdx.y * 256 + tid;
  for (int i = tid; i < kRowsIn * A; i += 256) {
    const int r = i / A, k = i % A;
    xs[r][k] = m0 + r < p.M ? p.x[(size_t)(m0 + r) * A + k] : 0.f;
  }
  __syncthreads();
  float acc[kRowsIn];
#pragma unroll
  for (int r = 0; r < kRowsIn; ++r) acc[r] = 0.f;
  constexpr int kK = 4;
#pragma unroll 1
  for (int k0 = 0; k0 < A; k0 += kK) {
    float wv[kK];
#pragma unroll
    for (int kk = 0; kk < kK; ++kk)
      wv[kk] = k0 + kk < A ? __uint_as_float((uint32_t)__ldg(p.w_in_t + (size_t)(k0 + kk) * d + n) << 16) : 0.f;
#pragma unroll
    for (int kk = 0; kk < kK; ++kk) {
      if (k0 + kk >= A) break;
#pragma unroll
      for (int r = 0; r < kRowsIn; ++r) acc[r] = fmaf(xs[r][k0 + kk], wv[kk], acc[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < kRowsIn; ++r) {
    const int m = m0 + r;
    if (m >= p.M) break;
    p.h[(size_t)m * d + n] = acc[r];
  }
}

// AdaRMSNorm after a residual GEMM (which added its branch into h), one warp
// per row: unless z is null, z = bf16(h rstd (1 + s) + b) in ACT128 (or E4M3
// codes with a row scale).
__global__ void __launch_bounds__(256) bresnorm_kernel(const __grid_constant__ BRowParams p) {
  grid_dep_launch();
  grid_dep_wait();
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= p.M) return;
  const int d = p.d, n4 = d / 128;   // float4 per lane
  const float4* hr = reinterpret_cast<const float4*>(p.h + (size_t)m * d);
  // every load of the row and of the modulation in flight before the first use
  float4 v[8], scv[8], shv[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool in = i < n4;
    v[i] = in ? hr[lane + 32 * i] : make_float4(0.f, 0.f, 0.f, 0.f);
    scv[i] = in ? *reinterpret_cast<const float4*>(p.s + 4 * (lane + 32 * i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    shv[i] = in ? *reinterpret_cast<const float4*>(p.b + 4 * (lane + 32 * i)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    s = fmaf(v[i].x, v[i].x, fmaf(v[i].y, v[i].y, fmaf(v[i].z, v[i].z, fmaf(v[i].w, v[i].w, s))));
  if (p.z == nullptr) return;
#pragma unroll
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float rs = 1.0f / sqrtf(s / (float)d + p.eps);
  if (p.zs == nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= n4) break;
      const int c = 4 * (lane + 32 * i);
      const float4 sc = scv[i];
      const float4 sh = shv[i];
      const uint32_t lo = pack2_bf16(fmaf(v[i].x * rs, 1.0f + sc.x, sh.x), fmaf(v[i].y * rs, 1.0f + sc.y, sh.y));
      const uint32_t hi = pack2_bf16(fmaf(v[i].z * rs, 1.0f + sc.z, sh.z), fmaf(v[i].w * rs, 1.0f + sc.w, sh.w));
      *reinterpret_cast<uint2*>(p.z + act128_off(m, c, d)) = make_uint2(lo, hi);
    }
    return;
  }
  // E4M3 z: y in fp32, the row's amax across the warp, codes of y / s_row
  float am = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= n4) break;
    const float4 sc = scv[i];
    const float4 sh = shv[i];
    v[i] = make_float4(fmaf(v[i].x * rs, 1.0f + sc.x, sh.x), fmaf(v[i].y * rs, 1.0f + sc.y, sh.y),
                       fmaf(v[i].z * rs, 1.0f + sc.z, sh.z), fmaf(v[i].w * rs, 1.0f + sc.w, sh.w));
    am = fmaxf(am, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float rq = act_rcp(am);
  if (lane == 0) p.zs[m] = act_scale(am);
  uint8_t* z8 = reinterpret_cast<uint8_t*>(p.z);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    if (i >= n4) break;
    const int c = 4 * (lane + 32 * i);
    *reinterpret_cast<uint32_t*>(z8 + act8_off(m, c, d)) = e4m3x4_of(v[i].x, v[i].y, v[i].z, v[i].w, rq);
  }
}

// R11 per-token E4M3 of a bf16 ACT128 matrix (attention output o, SwiGLU
// output u): one warp per row, lane i taking the pieces of 8 values at
// columns 8 (i + 32 j), K a multiple of 256 and at most 4096.  Two passes
// over the row: its amax, then the codes; the second read of the row comes
// from L2 (the matrix was just written and is at most 26 MB), which keeps
// the kernel small enough for many warps in flight per SM.
__global__ void __launch_bounds__(256) browquant_kernel(const __grid_constant__ BQuantParams p) {
  grid_dep_launch();
  grid_dep_wait();
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= p.M) return;
  const int np = p.K / 256;
  const uint16_t* src = p.src;
  float am = 0.f;
#pragma unroll 4
  for (int i = 0; i < np; ++i) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src + act128_off(m, 8 * (lane + 32 * i), p.K)));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      am = fmaxf(am, fmaxf(fabsf(__uint_as_float(w[q] << 16)), fabsf(__uint_as_float(w[q] & 0xFFFF0000u))));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  const float rq = act_rcp(am);
  if (lane == 0) p.scale[m] = act_scale(am);
#pragma unroll 4
  for (int i = 0; i < np; ++i) {
    const int c = 8 * (lane + 32 * i);
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src + act128_off(m, c, p.K)));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2];
#pragma unroll
    for (int q = 0; q < 2; ++q)
      out[q] = e4m3x4_of(__uint_as_float(w[2 * q] << 16), __uint_as_float(w[2 * q] & 0xFFFF0000u),
                         __uint_as_float(w[2 * q + 1] << 16), __uint_as_float(w[2 * q + 1] & 0xFFFF0000u), rq);
    *reinterpret_cast<uint2*>(p.dst + act8_off(m, c, p.K)) = make_uint2(out[0], out[1]);
  }
}

// Final AdaRMSNorm + out-proj + Euler: 16 rows per CTA (8 warps).  The rows'
// normalised activations y stay in shared memory (fp32); warp w evaluates
// actions a = w, w + 8, ...: lanes split the d inputs (coalesced W_out row),
// 16 row sums reduced by shuffles.
__global__ void __launch_bounds__(256) boutproj_kernel(const __grid_constant__ BRowParams p) {
  extern __shared__ float ys[];   // [kRowsIn][d]
  grid_dep_launch();
  grid_dep_wait();
  const int m0 = blockIdx.x * kRowsIn;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = p.d, A = p.A;
  // final norm of the block's rows: lane i holds float4 columns 4 (i + 32 j),
  // all loads in flight before the reduction (d a multiple of 128, <= 1024)
  const int n4 = d / 128;
  for (int r = warp; r < kRowsIn; r += 8) {
    const int m = m0 + r;
    float4* y = reinterpret_cast<float4*>(ys + (size_t)r * d);
    const bool row_ok = m < p.M;
    const float4* hr = reinterpret_cast<const float4*>(p.h + (size_t)(row_ok ? m : 0) * d);
    float4 v[8], scv[8], shv[8];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const bool in = i < n4;
      v[i] = in && row_ok ? hr[lane + 32 * i] : make_float4(0.f, 0.f, 0.f, 0.f);
      scv[i] = in ? *reinterpret_cast<const float4*>(p.s + 4 * (lane + 32 * i)) : make_float4(0.f, 0.f, 0.f, 0.f);
      shv[i] = in ? *reinterpret_cast<const float4*>(p.b + 4 * (lane + 32 * i)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      s = fmaf(v[i].x, v[i].x, fmaf(v[i].y, v[i].y, fmaf(v[i].z, v[i].z, fmaf(v[i].w, v[i].w, s))));
#pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float rs = 1.0f / sqrtf(s / (float)d + p.eps);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i >= n4) break;
      y[lane + 32 * i] = row_ok ? make_float4(fmaf(v[i].x * rs, 1.0f + scv[i].x, shv[i].x),
                                              fmaf(v[i].y * rs, 1.0f + scv[i].y, shv[i].y),
                                              fmaf(v[i].z * rs, 1.0f + scv[i].z, shv[i].z),
                                              fmaf(v[i].w * rs, 1.0f + scv[i].w, shv[i].w))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();
  for (int a = warp; a < A; a += 8) {
    const uint16_t* w = p.w_out + (size_t)a * d;
    float acc[kRowsIn];
#pragma unroll
    for (int r = 0; r < kRowsIn; ++r) acc[r] = 0.f;
    // 8 weights in flight per lane per iteration (L2 hits)
    constexpr int kU = 8;
#pragma unroll 1
    for (int c0 = lane; c0 < d; c0 += 32 * kU) {
      float wv[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        wv[u] = c0 + 32 * u < d ? __uint_as_float((uint32_t)__ldg(w + c0 + 32 * u) << 16) : 0.f;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int c = c0 + 32 * u;
        if (c >= d) break;
#pragma unroll
        for (int r = 0; r < kRowsIn; ++r) acc[r] = fmaf(ys[(size_t)r * d + c], wv[u], acc[r]);
      }
    }
#pragma unroll
    for (int r = 0; r < kRowsIn; ++r)
#pragma unroll
      for (int o = 16; o; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
    if (lane < kRowsIn) {
      float v = 0.f;
#pragma unroll
      for (int r = 0; r < kRowsIn; ++r)
        if (r == lane) v = acc[r];
      const int m = m0 + lane;
      if (m < p.M) {
        if (p.out_bias != nullptr) v += p.out_bias[a];
        p.v_out[(size_t)m * A + a] = v;
        if (p.x_out != nullptr) p.x_out[(size_t)m * A + a] += p.dt * v;
      }
    }
  }
}

// ------------------------------------------------------------------ attention
// One CTA per (request b, KV group g, block of 64 of the group's G*T query
// rows); 4 warps x 16 rows.  Each warp keeps its q rows as mma.sync A
// fragments in registers (loaded once from global), and walks the keys in
// tiles of 64 (K and V double-buffered in shared memory by bulk copy):
// S = q K^T for the 64 keys (m16n8k16), one online-softmax update per tile
// (base 2), then P V with P taken straight from the S accumulators.
constexpr int kAttnKeys = 64;
template <int HD>
__global__ void __launch_bounds__(128, 3) battn_kernel(const __grid_constant__ BAttnParams p) {
  constexpr int KSTEPS = HD / 16;
  constexpr int DT = HD / 8;                      // 8-column tiles of the output
  constexpr int NT = kAttnKeys / 8;               // 8-key tiles of S
  constexpr int TILE = kAttnKeys * HD * 2;        // bytes of one K or V tile
  extern __shared__ uint8_t sm_raw[];
  uint8_t* sm = align1024(sm_raw);
  uint8_t* kbuf = sm;                             // [2] K tiles
  uint8_t* vbuf = sm + 2 * TILE;                  // [2] V tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(vbuf + 2 * TILE);   // [2] tile barriers
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  grid_dep_launch();
  grid_dep_wait();
  const int qb = blockIdx.x % p.qblocks;
  const int g = (blockIdx.x / p.qblocks) % p.Hkv;
  const int b = blockIdx.x / (p.qblocks * p.Hkv);
  const int G = p.Hq / p.Hkv, T = p.T;
  const int P = p.P_dev[b];
  const int S = P + T;
  const int row0 = qb * 64;
  const int nrows = min(64, G * T - row0);
  if (nrows <= 0) return;
  const size_t kvoff = (((size_t)b * p.Hkv + g) * p.S_max) * HD;
  const uint16_t* kg = p.kc + kvoff;
  const uint16_t* vg = p.vc + kvoff;
  const int ntile = (S + kAttnKeys - 1) / kAttnKeys;
  if (tid == 0) {
    mbar_init(smem_u32(&bars[0]), 1);
    mbar_init(smem_u32(&bars[1]), 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t pol = policy_evict_last();
  auto issue = [&](int it) {
    const int kb = it * kAttnKeys, nk = min(kAttnKeys, S - kb);
    const uint32_t bar = smem_u32(&bars[it & 1]);
    mbar_arrive_expect_tx(bar, 2u * (uint32_t)nk * HD * 2u);
    bulk_g2s(smem_u32(kbuf + (it & 1) * TILE), kg + (size_t)kb * HD, (uint32_t)nk * HD * 2, bar, pol);
    bulk_g2s(smem_u32(vbuf + (it & 1) * TILE), vg + (size_t)kb * HD, (uint32_t)nk * HD * 2, bar, pol);
  };
  if (tid == 0) {
    issue(0);
    if (ntile > 1) issue(1);
  }
  // q fragments (rows r0 + gid, r0 + gid + 8; columns 16 kk + 2 tig (+8))
  const int gid = lane >> 2, tig = lane & 3;
  const int r0 = 16 * warp;
  uint32_t qa[KSTEPS][4];
  {
    const uint16_t* qg = p.qbuf + (((size_t)b * p.Hkv + g) * p.q_rows) * HD;
    const int Ra = row0 + r0 + gid, Rb = Ra + 8;   // rows of the group block (q_rows padding is zero)
    const uint16_t* qra = qg + (size_t)Ra * HD;
    const uint16_t* qrb = qg + (size_t)Rb * HD;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int e0 = 16 * kk + 2 * tig;
      qa[kk][0] = *reinterpret_cast<const uint32_t*>(qra + ((((e0 >> 3)) ^ (Ra & 7)) << 3) + (e0 & 7));
      qa[kk][1] = *reinterpret_cast<const uint32_t*>(qrb + ((((e0 >> 3)) ^ (Rb & 7)) << 3) + (e0 & 7));
      qa[kk][2] = *reinterpret_cast<const uint32_t*>(qra + ((((e0 >> 3) + 1) ^ (Ra & 7)) << 3) + (e0 & 7));
      qa[kk][3] = *reinterpret_cast<const uint32_t*>(qrb + ((((e0 >> 3) + 1) ^ (Rb & 7)) << 3) + (e0 & 7));
    }
  }
  const long long budget = p.spin_budget;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  const int kkey = (lane & 7) + ((lane >> 4) << 3);
  const int k_pc = (lane >> 3) & 1;
  const int vkey = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int v_pc = lane >> 4;
  bool good = true;
#pragma unroll 1
  for (int it = 0; it < ntile; ++it) {
    const int kb = it * kAttnKeys, nk = min(kAttnKeys, S - kb);
    if (!mbar_wait(smem_u32(&bars[it & 1]), (it >> 1) & 1, budget)) {
      atomicOr(p.err, 0x2000u);
      good = false;
      break;
    }
    uint8_t* ks_ = kbuf + (it & 1) * TILE;
    uint8_t* vs_ = vbuf + (it & 1) * TILE;
    if (nk < kAttnKeys) {
      // zero V rows past the last key so no stale shared memory meets a zero weight
      uint4* zr = reinterpret_cast<uint4*>(vs_ + (size_t)nk * HD * 2);
      for (int i = tid; i < (kAttnKeys - nk) * HD * 2 / 16; i += 128) zr[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
    }
    const uint32_t ka = smem_u32(ks_), va = smem_u32(vs_);
    // S = q K^T over the 64 keys of the tile (kb is a multiple of 64, so a
    // key's swizzle row is its index inside the tile)
    float sc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
      for (int j2 = 0; j2 < NT / 2; ++j2) {
        const int key = 16 * j2 + kkey;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ka + key * HD * 2 + (((2 * kk + k_pc) ^ (key & 7)) << 4), b0, b1, b2, b3);
        mma16816(sc[2 * j2], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
        mma16816(sc[2 * j2 + 1], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b2, b3);
      }
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < NT; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = 8 * j + 2 * tig + (e & 1);
        sc[j][e] = key < nk ? sc[j][e] * sl2 : -INFINITY;
        mx[e >> 1] = fmaxf(mx[e >> 1], sc[j][e]);
      }
    }
    float corr[2], mnew[2], ls[2] = {0.f, 0.f};
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
      mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
      mnew[h2] = fmaxf(m_r[h2], mx[h2]);
      corr[h2] = (m_r[h2] == -INFINITY) ? 0.f : exp2f(m_r[h2] - mnew[h2]);
      m_r[h2] = mnew[h2];
    }
    uint32_t pa[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const float p0 = exp2f(sc[j][0] - mnew[0]), p1 = exp2f(sc[j][1] - mnew[0]);
      const float p2 = exp2f(sc[j][2] - mnew[1]), p3 = exp2f(sc[j][3] - mnew[1]);
      ls[0] += p0 + p1;
      ls[1] += p2 + p3;
      pa[j][0] = pack2_bf16(p0, p1);
      pa[j][1] = pack2_bf16(p2, p3);
    }
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      ls[h2] += __shfl_xor_sync(0xffffffffu, ls[h2], 1);
      ls[h2] += __shfl_xor_sync(0xffffffffu, ls[h2], 2);
      l_r[h2] = l_r[h2] * corr[h2] + ls[h2];
    }
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= corr[0];
      o[i][1] *= corr[0];
      o[i][2] *= corr[1];
      o[i][3] *= corr[1];
    }
    // O += P V, 16 keys at a time (A fragment = the S accumulators of two 8-key tiles)
#pragma unroll
    for (int j2 = 0; j2 < NT / 2; ++j2) {
      const int key = 16 * j2 + vkey;
      const uint32_t v_lane = va + key * HD * 2;
#pragma unroll
      for (int i = 0; i < DT; i += 2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(v_lane + (((i + v_pc) ^ (key & 7)) << 4), b0, b1, b2, b3);
        mma16816(o[i], pa[2 * j2][0], pa[2 * j2][1], pa[2 * j2 + 1][0], pa[2 * j2 + 1][1], b0, b1);
        mma16816(o[i + 1], pa[2 * j2][0], pa[2 * j2][1], pa[2 * j2 + 1][0], pa[2 * j2 + 1][1], b2, b3);
      }
    }
    // the buffer is refilled with tile it + 2 once every warp is done with it
    __syncthreads();
    if (tid == 0 && it + 2 < ntile) {
      fence_proxy_async_smem();
      issue(it + 2);
    }
  }
  if (!good) return;
  // normalise and store o rows: query row R -> head g*G + R / T, token R % T
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int R = row0 + r0 + gid + 8 * h2;
    if (R - row0 >= nrows) continue;
    const float inv = 1.0f / l_r[h2];
    const int head = g * G + R / T, t = R % T;
    const int m = b * T + t;
    const int K = p.Hq * HD;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      const int c = head * HD + 8 * i + 2 * tig;
      *reinterpret_cast<uint32_t*>(p.o_act + act128_off(m, c, K)) =
          pack2_bf16(o[i][2 * h2] * inv, o[i][2 * h2 + 1] * inv);
    }
  }
}

// Launch with programmatic stream serialization: the kernel may start while
// the previous one in the stream finishes (it waits with griddepcontrol.wait
// before touching what that kernel writes).
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), int grid, int block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(block, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int BN, int EPI, bool F8>
cudaError_t launch_bgemm_t(const BGemmParams& p, int n_sms, cudaStream_t st) {
  using C = BCfg<BN>;
  static_assert(C::kSmem <= 232448, "bgemm shared memory exceeds the per-block limit");
  cudaError_t e = cudaFuncSetAttribute(bgemm_kernel<BN, EPI, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)C::kSmem);
  if (e != cudaSuccess) return e;
  const int ntiles = (p.Mp / kBM) * (p.N / BN);
  const int grid = ntiles < n_sms ? ntiles : n_sms;
  return launch_pdl(bgemm_kernel<BN, EPI, F8>, grid, kBThreads, C::kSmem, st, p);
}

template <bool F8>
cudaError_t launch_bgemm_f(const BGemmParams& p, int epi, int bn, int n_sms, cudaStream_t st) {
  if (epi == BE_RESID)
    return bn == 256 ? launch_bgemm_t<256, BE_RESID, F8>(p, n_sms, st) : launch_bgemm_t<128, BE_RESID, F8>(p, n_sms, st);
  if (epi == BE_SWIGLU) return launch_bgemm_t<256, BE_SWIGLU, F8>(p, n_sms, st);
  return bn == 256 ? launch_bgemm_t<256, BE_QKV, F8>(p, n_sms, st) : launch_bgemm_t<128, BE_QKV, F8>(p, n_sms, st);
}

}  // namespace

// 256-wide weight tiles wherever N allows: per k-block a CTA then moves 48 KB
// of operands for 128 x 256 x 64 MACs instead of 32 KB for 128 x 128 x 64,
// which matters because the operand stream from L2 is what bounds these GEMMs.
int bgemm_bn(int epi, int N) {
  if (epi == BE_SWIGLU) return 256;
  return N % 256 == 0 ? 256 : 128;
}

// E4M3 operands when p.a_scale is set (W8A8), bf16 otherwise.
cudaError_t launch_bgemm(const BGemmParams& p, int epi, int n_sms, cudaStream_t st) {
  const int bn = bgemm_bn(epi, p.N);
  return p.a_scale != nullptr ? launch_bgemm_f<true>(p, epi, bn, n_sms, st)
                              : launch_bgemm_f<false>(p, epi, bn, n_sms, st);
}

// Row-major bf16 [M][K] -> ACT128 [Mp/128][K/64]; rows M .. Mp-1 are zero.
__global__ void rows_to_act128_kernel(const uint16_t* __restrict__ src, int M, int Mp, int K,
                                      uint16_t* __restrict__ dst) {
  const int pieces = K / 8;
  const size_t total = (size_t)Mp * pieces;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int m = (int)(i / pieces), c = (int)(i % pieces) * 8;
    const uint4 v = m < M ? *reinterpret_cast<const uint4*>(src + (size_t)m * K + c) : make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(dst + act128_off(m, c, K)) = v;
  }
}

cudaError_t launch_rows_to_act128(const uint16_t* src, int M, int Mp, int K, uint16_t* dst, cudaStream_t st) {
  rows_to_act128_kernel<<<1024, 256, 0, st>>>(src, M, Mp, K, dst);
  return cudaGetLastError();
}

cudaError_t launch_binproj(const BRowParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3((p.M + kRowsIn - 1) / kRowsIn, p.d / 256, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, binproj_kernel, p);
}

cudaError_t launch_bresnorm(const BRowParams& p, cudaStream_t st) {
  return launch_pdl(bresnorm_kernel, (p.M + 7) / 8, 256, 0, st, p);
}

cudaError_t launch_browquant(const BQuantParams& p, cudaStream_t st) {
  return launch_pdl(browquant_kernel, (p.M + 7) / 8, 256, 0, st, p);
}

cudaError_t launch_boutproj(const BRowParams& p, cudaStream_t st) {
  const size_t smem = (size_t)kRowsIn * p.d * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(boutproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(boutproj_kernel, (p.M + kRowsIn - 1) / kRowsIn, 256, smem, st, p);
}

cudaError_t launch_battn(const BAttnParams& p, cudaStream_t st) {
  const size_t smem = 1024 + (size_t)4 * kAttnKeys * p.hd * 2 + 64;
  const int grid = p.B * p.Hkv * p.qblocks;
  cudaError_t e;
  if (p.hd == 128) {
    e = cudaFuncSetAttribute(battn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(battn_kernel<128>, grid, 128, smem, st, p);
  } else {
    e = cudaFuncSetAttribute(battn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(battn_kernel<64>, grid, 128, smem, st, p);
  }
  return e;
}

}  // namespace fm
