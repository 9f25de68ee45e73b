// Time conditioning, once per call for every Euler time t_k = 1 - k/n:
//   e_k = sinusoid256(t_k)  (periods geometric from 4e-3 to 4, sin then cos)
//   h1  = SiLU(e W1^T)      -> bf16, ACT64 rows k
//   m_k = h1 W2^T           -> fp32 [n, L*6d + 2d]
// "LingBot-VLA on Thor (sm_110)", §2 Build names the fused AdaRMSNorm these
// rows modulate; the two-linear SiLU MLP and the period range are this
// library's reading (the pages give no formula).
//
// time_gemm_kernel is a persistent, warp-specialised tcgen05 GEMM with M = 64
// (steps, zero-padded), N = 128 channels per tile, K = d: warp 0 streams
// packed W2 tiles through a 6-stage shared-memory ring with bulk copies,
// warp 1 issues tcgen05.mma into one of two TMEM accumulators, warps 2-5
// drain the other accumulator to global memory.  It is a pure weight stream
// (457.7 MB at d = 1024, L = 36), so it is sized to keep HBM busy.
#include <cuda_bf16.h>
#include <cstdint>

#include "fm_internal.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {
constexpr int kTStages = 6;
constexpr int kTTile = 128;                  // channels per tile
constexpr uint32_t kTChunk = kTTile * 128;   // 16 KB: 128 rows x 64 bf16
constexpr double kTwoPi = 6.283185307179586476925286766559;
}  // namespace

// Hidden rows of the time MLP: e_k (fp64 -> fp32) for every step in shared
// memory, then one warp per hidden unit i: lanes split W1[i, :] (coalesced)
// and h1[k, i] = SiLU(sum_j e_k[j] W1[i, j]) for all steps k, stored bf16 in
// ACT64 row k.
__global__ void time_embed_kernel(const __grid_constant__ TimeParams p) {
  extern __shared__ float e_dyn[];   // [n_steps][kTimeDim]
  float (*e)[kTimeDim] = reinterpret_cast<float (*)[kTimeDim]>(e_dyn);
  const int half = kTimeDim / 2;
  for (int idx = threadIdx.x; idx < p.n_steps * half; idx += blockDim.x) {
    const int k = idx / half, j = idx % half;
    const double t = 1.0 - (double)k / (double)p.n_steps;
    const double period = 4e-3 * pow(4.0 / 4e-3, (double)j / (double)(half - 1));
    const double ang = kTwoPi * t / period;
    e[k][j] = (float)sin(ang);
    e[k][j + half] = (float)cos(ang);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int i = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (i >= p.d) return;
  // lane holds W1[i, 8*lane .. 8*lane+7]
  const uint4 wv = *reinterpret_cast<const uint4*>(p.w1 + (size_t)i * kTimeDim + 8 * lane);
  const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
  float w[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    w[2 * q] = __uint_as_float(wr[q] << 16);
    w[2 * q + 1] = __uint_as_float(wr[q] & 0xFFFF0000u);
  }
  const int kb = i >> 6, c = (i & 63) >> 3;
  for (int k = 0; k < p.n_steps; ++k) {
    float acc = 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) acc = fmaf(e[k][8 * lane + q], w[q], acc);
#pragma unroll
    for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float h = acc / (1.0f + expf(-acc));
      uint16_t* row = p.h1_act + (size_t)kb * (kRows * 64) + (size_t)k * 64;
      __nv_bfloat16 hb = __float2bfloat16_rn(h);
      row[((c ^ (k & 7)) << 3) + (i & 7)] = *reinterpret_cast<uint16_t*>(&hb);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) time_gemm_kernel(const __grid_constant__ TimeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nkb = p.d / 64;
  uint8_t* A = smem;
  uint8_t* ring = A + (size_t)nkb * 8192;
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + kTStages * kTChunk);
  uint64_t* full = bars;                 // [kTStages]
  uint64_t* empty = bars + kTStages;     // [kTStages]
  uint64_t* a_full = bars + 2 * kTStages;
  uint64_t* tfull = a_full + 1;          // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (p.n_mod + kTTile - 1) / kTTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTStages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(a_full), 1);
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull[a]), 1);
      mbar_init(smem_u32(&tempty[a]), kComputeWarps);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long budget = p.spin_budget;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      mbar_arrive_expect_tx(smem_u32(a_full), (uint32_t)nkb * 8192u);
      for (int kb = 0; kb < nkb; ++kb)
        bulk_g2s(smem_u32(A + (size_t)kb * 8192), p.h1_act + (size_t)kb * kRows * 64, 8192,
                 smem_u32(a_full), pol_a);
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const uint32_t s = it % kTStages, ph = (it / kTStages) & 1;
          if (it >= kTStages && !mbar_wait(smem_u32(&empty[s]), ph ^ 1, budget)) {
            atomicOr(p.err, 0x1u);
            goto producer_done;
          }
          mbar_arrive_expect_tx(smem_u32(&full[s]), kTChunk);
          bulk_g2s(smem_u32(ring + s * kTChunk),
                   p.w2_packed + ((size_t)tile * nkb + kb) * kTChunk, kTChunk,
                   smem_u32(&full[s]), pol_w);
        }
      }
      // Drain: every issued copy must land before the CTA may exit.
      for (uint32_t j = (it > kTStages ? it - kTStages : 0); j < it; ++j)
        mbar_wait(smem_u32(&full[j % kTStages]), (j / kTStages) & 1, budget);
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kRows, kTTile);
      bool ok = mbar_wait(smem_u32(a_full), 0, budget);
      if (!ok) atomicOr(p.err, 0x2u);
      uint32_t it = 0, local = 0;
      for (int tile = blockIdx.x; ok && tile < ntiles; tile += gridDim.x, ++local) {
        const uint32_t acc = local & 1;
        if (local >= 2 && !mbar_wait(smem_u32(&tempty[acc]), ((local >> 1) - 1) & 1, budget)) {
          atomicOr(p.err, 0x4u);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kTTile;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const uint32_t s = it % kTStages, ph = (it / kTStages) & 1;
          if (!mbar_wait(smem_u32(&full[s]), ph, budget)) {
            atomicOr(p.err, 0x8u);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(A + (size_t)kb * 8192);
          const uint32_t b_base = smem_u32(ring + s * kTChunk);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_bf16(d_tmem, desc_sw128(a_base + k16 * 32), desc_sw128(b_base + k16 * 32), idesc,
                     (kb | k16) != 0);
          mma_commit(smem_u32(&empty[s]));
        }
        if (ok) mma_commit(smem_u32(&tfull[acc]));
      }
    }
  } else {
    // Epilogue warps 2..5: warp w reads TMEM lanes 32*(w%4) .. +15, i.e.
    // accumulator rows 16*(w%4) .. +15 (M = 64 layout).
    const int sp = warp & 3;
    const int row = 16 * sp + lane;
    const bool row_ok = lane < 16 && row < p.n_steps;
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++local) {
      const uint32_t acc = local & 1;
      if (!mbar_wait(smem_u32(&tfull[acc]), (local >> 1) & 1, budget)) {
        atomicOr(p.err, 0x10u);
        break;
      }
      tc_fence_after();
      const uint32_t t_base = tmem + ((uint32_t)(32 * sp) << 16) + acc * kTTile;
      float* out = p.mod + (size_t)row * p.n_mod + (size_t)tile * kTTile;
#pragma unroll 1
      for (int cb = 0; cb < kTTile / 16; ++cb) {
        float v[16];
        tmem_ld16(t_base + cb * 16, v);
        tmem_ld_wait();
        if (row_ok) {
          const int col0 = tile * kTTile + cb * 16;
          if (col0 + 16 <= p.n_mod) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              *reinterpret_cast<float4*>(out + cb * 16 + 4 * q) =
                  make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          } else {
            for (int q = 0; q < 16; ++q)
              if (col0 + q < p.n_mod) out[cb * 16 + q] = v[q];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&tempty[acc]));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t time_gemm_smem_bytes(int d) {
  return 1024 + (size_t)(d / 64) * 8192 + kTStages * kTChunk + 256;
}

cudaError_t launch_time(const TimeParams& p, int n_sms, cudaStream_t st) {
  const size_t esmem = (size_t)p.n_steps * kTimeDim * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(time_embed_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)esmem);
  if (e != cudaSuccess) return e;
  time_embed_kernel<<<(p.d + 7) / 8, 256, esmem, st>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = time_gemm_smem_bytes(p.d);
  e = cudaFuncSetAttribute(time_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int ntiles = (p.n_mod + kTTile - 1) / kTTile;
  const int grid = ntiles < n_sms ? ntiles : n_sms;
  time_gemm_kernel<<<grid, kThreads, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace fm
