// Batched GQA attention on the 5th-generation tensor cores ("LingBot-VLA on
// Thor (sm_110)", §3 FlashAttention-4: the denoise attention is grouped-query
// attention over the cached prefix keys and the chunk's own keys, pack_gqa).
//
// One CTA per (request b, KV group g, block of 128 query rows of that group:
// row (h % G) T + t for the group's G heads and the chunk's T tokens), eight
// warps; query row i (TMEM lane i of the M = 128 accumulators) belongs to lane
// i % 32 of warps i / 32 and i / 32 + 4, which split its keys and columns.
// Two CTAs share an SM (256 TMEM columns and ~99 KB of shared memory each), so
// one CTA's loads and tensor-core work overlap the other's softmax.
//   1. Thread 0 moves Q rows and, per 128-key chunk, K and V rows into shared
//      memory with one TMA copy per 64-element half of 128 rows (4-D views
//      (64 elements, half, row, segment) of the q buffer and the caches): both
//      store each row's 16-byte pieces swizzled by (row & 7), so every 128-byte
//      half row is already a row of the 128-byte-swizzled image tcgen05 reads,
//      and the copy lands as [half][128 rows][128 B].
//   2. Pass 1, per chunk: S = Q K^T into TMEM columns [0, 128) (K is the
//      K-major B operand); each thread reads its half of the chunk's S row
//      and keeps the running row maximum.  The two halves meet in shared
//      memory: m = the row maximum over every key.
//   3. Pass 2, per chunk: S = Q K^T again (a 128-key MMA costs ~0.25 us), p =
//      exp2(s log2(e) / sqrt(hd) - m) for valid keys (0 for the padding keys
//      of the last chunk) in bf16 into the K-major image of P (over K, which
//      the MMA has finished with), l += p in fp32, then O += P V in TMEM
//      columns [128, 128 + hd); V rows, hd contiguous, are the MN-major B
//      operand as they arrive.  The maximum is final before any p is formed,
//      so the softmax is exact and O is never rescaled.
//   4. o = O / l in bf16 goes to the ACT128 activation of o_proj.
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

#include "fm_batch.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {

constexpr int kAtThreads = 256;          // 8 warps: two per TMEM lane quarter
constexpr int kAtRows = 128;            // query rows per CTA (MMA M)
constexpr int kAtChunk = 128;           // keys per chunk (MMA N of S, K of O)
constexpr int kAtMaxChunks = 3;
constexpr int kAtTile = kAtRows * 128;  // bytes of one 128-row x 128-byte image
constexpr int kOCol = kAtChunk;         // first TMEM column of O (S takes [0, 128))
constexpr int kAtTmem = 256;            // TMEM columns per CTA (two CTAs per SM)

// Barriers: Q loaded, K chunk loaded, V chunk loaded, S MMA done, PV MMA done
// (each completes once per use; waits alternate parity).
enum { BQ = 0, BK = 1, BV = 2, BS = 3, BO = 4, kAtBars = 5 };

template <int HD>
struct AtCfg {
  static constexpr int kImg = (HD / 64) * kAtTile;          // Q / K / V image: [half][128 rows][128 B]
  static constexpr int kPBytes = 2 * kAtTile;               // P chunk: [key half][128 rows][128 B]
  static constexpr int kKP = kImg > kPBytes ? kImg : kPBytes;   // K chunk, then P of that chunk
  static constexpr int kSmem = 1024 + kImg + kKP + kImg + 256 + 2 * 2 * kAtRows * 4;
};

__device__ __forceinline__ uint32_t pk_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// One TMA copy per 64-element half of rows [row0, row0 + 128) of segment
// `seg` of a (64, half, row, segment) view -> image dst[half][128 rows][128 B].
template <int HD>
__device__ __forceinline__ void tma_tile(uint8_t* dst, const CUtensorMap* tm, int row0, int seg, uint32_t bar,
                                         uint64_t pol) {
  mbar_arrive_expect_tx(bar, (uint32_t)(HD / 64) * kAtTile);
#pragma unroll
  for (int h = 0; h < HD / 64; ++h) tma_load_4d(smem_u32(dst + h * kAtTile), tm, 0, h, row0, seg, bar, pol);
}

}  // namespace

template <int HD>
__global__ void __launch_bounds__(kAtThreads, 2) battn_tc_kernel(const __grid_constant__ BAttnParams p) {
  using C = AtCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = sm;
  uint8_t* kp = sm + C::kImg;                          // K chunk, then P of that chunk
  uint8_t* vs = sm + C::kImg + C::kKP;
  uint64_t* bars = reinterpret_cast<uint64_t*>(vs + C::kImg);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + kAtBars + 1);
  float* red = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + 256);   // [2 halves][128 rows]
  const int tid = threadIdx.x, warp = tid >> 5;
  const int half = warp >> 2, row = 32 * (warp & 3) + (tid & 31);   // row = TMEM lane
  const int qb = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv, T = p.T;
  const int nq = G * T;                                // query rows of the group
  const long long budget = p.spin_budget;

  if (tid == 0) {
    for (int i = 0; i < kAtBars; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), kAtTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  grid_dep_wait();   // q and the chunk's cache rows come from the QKV GEMM

  const int S = p.P_dev[b] + T;                       // keys of this request
  const int nch = (S + kAtChunk - 1) / kAtChunk;
  const int qseg = b * p.Hkv + g, kvseg = p.seg_base + qseg;
  // K and V rows serve the group's other query blocks too: keep them in L2
  const uint64_t pol_q = policy_evict_first(), pol_kv = policy_evict_last();
  const uint32_t id_s = idesc_bf16(kAtRows, kAtChunk), id_o = idesc_bf16_bmn(kAtRows, HD);
  const uint32_t trow = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  const int cb = half * (kAtChunk / 2);                // this thread's 64 columns of a chunk
  bool ok = true;

  if (tid == 0) {
    tma_tile<HD>(qs, &p.tm_q, qb * kAtRows, qseg, smem_u32(&bars[BQ]), pol_q);
    tma_tile<HD>(kp, &p.tm_k, 0, kvseg, smem_u32(&bars[BK]), pol_kv);
    tma_tile<HD>(vs, &p.tm_v, 0, kvseg, smem_u32(&bars[BV]), pol_kv);
  }
  __syncwarp();

  float mx = -INFINITY, mb = 0.f, l = 0.f;
  for (int i = 0; i < 2 * nch; ++i) {
    const int c = i < nch ? i : i - nch;
    const bool second = i >= nch;
    // S = Q K_c^T
    if (tid == 32) {
      if (i == 0) ok &= mbar_wait(smem_u32(&bars[BQ]), 0, budget);
      ok &= mbar_wait(smem_u32(&bars[BK]), (uint32_t)(i & 1), budget);
      tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < HD / 16; ++k16) {
        const uint32_t off = (uint32_t)((k16 >> 2) * kAtTile + (k16 & 3) * 32);
        mma_bf16(tmem, desc_sw128(smem_u32(qs) + off), desc_sw128(smem_u32(kp) + off), id_s, k16 > 0);
      }
      mma_commit(smem_u32(&bars[BS]));
    }
    __syncwarp();
    ok &= mbar_wait(smem_u32(&bars[BS]), (uint32_t)(i & 1), budget);
    tc_fence_after();
    const int k0 = c * kAtChunk + cb;                  // key index of this thread's first column
    if (!second) {
      // pass 1: running maximum over valid keys
#pragma unroll 1
      for (int j0 = 0; j0 < kAtChunk / 2; j0 += 32) {
        float v[2][16];
        tmem_ld16(trow + cb + j0, v[0]);
        tmem_ld16(trow + cb + j0 + 16, v[1]);
        tmem_ld_wait();
        if (k0 + j0 + 32 <= S) {
#pragma unroll
          for (int j = 0; j < 32; ++j) mx = fmaxf(mx, v[j >> 4][j & 15]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (k0 + j0 + j < S) mx = fmaxf(mx, v[j >> 4][j & 15]);
        }
      }
      tc_fence_before();
      __syncthreads();   // S read: the next S MMA may overwrite it, the K buffer is free
      if (tid == 0) {
        // the next K chunk (pass 2 starts again at chunk 0)
        tma_tile<HD>(kp, &p.tm_k, (c + 1 < nch ? c + 1 : 0) * kAtChunk, kvseg, smem_u32(&bars[BK]), pol_kv);
      }
      if (c == nch - 1) {
        red[half * kAtRows + row] = mx;
        __syncthreads();
        mb = fmaxf(red[row], red[kAtRows + row]) * sl2;
      }
      continue;
    }
    // pass 2: p = exp2(s sl2 - m) -> P (over the K buffer), l += p
#pragma unroll 1
    for (int j0 = 0; j0 < kAtChunk / 2; j0 += 32) {
      float v[2][16];
      tmem_ld16(trow + cb + j0, v[0]);
      tmem_ld16(trow + cb + j0 + 16, v[1]);
      tmem_ld_wait();
      uint32_t pk[16];
      if (k0 + j0 + 32 <= S) {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float e0 = exp2f(fmaf(v[(2 * j) >> 4][(2 * j) & 15], sl2, -mb));
          const float e1 = exp2f(fmaf(v[(2 * j + 1) >> 4][(2 * j + 1) & 15], sl2, -mb));
          l += e0;
          l += e1;
          pk[j] = pk_bf16(e0, e1);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float s0 = v[(2 * j) >> 4][(2 * j) & 15], s1 = v[(2 * j + 1) >> 4][(2 * j + 1) & 15];
          const float e0 = k0 + j0 + 2 * j < S ? exp2f(fmaf(s0, sl2, -mb)) : 0.f;
          const float e1 = k0 + j0 + 2 * j + 1 < S ? exp2f(fmaf(s1, sl2, -mb)) : 0.f;
          l += e0;
          l += e1;
          pk[j] = pk_bf16(e0, e1);
        }
      }
      // columns cb + j0 .. + 31 of the chunk: key half (cb + j0) / 64, pieces ((cb + j0) % 64) / 8 .. + 3
      const int col = cb + j0, kh = col >> 6, pc0 = (col & 63) >> 3;
      uint8_t* prow = kp + kh * kAtTile + row * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(prow + (((pc0 + q) ^ (row & 7)) << 4)) =
            make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();   // P complete, S read
    if (tid == 32) {
      ok &= mbar_wait(smem_u32(&bars[BV]), (uint32_t)(c & 1), budget);
      tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < kAtChunk / 16; ++k16) {
        const uint32_t aoff = (uint32_t)((k16 >> 2) * kAtTile + (k16 & 3) * 32);
        mma_bf16(tmem + kOCol, desc_sw128(smem_u32(kp) + aoff),
                 desc_sw128_mn(smem_u32(vs) + (uint32_t)k16 * 2048u, kAtTile), id_o, (c | k16) != 0);
      }
      mma_commit(smem_u32(&bars[BO]));
    }
    __syncwarp();
    if (tid == 0 && c + 1 < nch) {
      // the P and V buffers are free once this chunk's PV MMAs are done
      ok &= mbar_wait(smem_u32(&bars[BO]), (uint32_t)(c & 1), budget);
      tma_tile<HD>(kp, &p.tm_k, (c + 1) * kAtChunk, kvseg, smem_u32(&bars[BK]), pol_kv);
      tma_tile<HD>(vs, &p.tm_v, (c + 1) * kAtChunk, kvseg, smem_u32(&bars[BV]), pol_kv);
    }
    __syncwarp();
  }
  ok &= mbar_wait(smem_u32(&bars[BO]), (uint32_t)((nch - 1) & 1), budget);
  tc_fence_after();
  red[half * kAtRows + row] = l;
  __syncthreads();
  l = red[row] + red[kAtRows + row];

  // 4: o = O / l -> ACT128 [Mp/128][Hq*hd/64] rows b T + t, columns h hd + e;
  // each thread of the row takes half of the hd columns
  const int qr = qb * kAtRows + row;
  const float inv = 1.0f / l;
  const int head = g * G + (qr < nq ? qr / T : 0), t = qr < nq ? qr % T : 0;
  const int m = b * T + t;
  const int K = p.Hq * HD;
  for (int e0 = half * (HD / 2); e0 < (half + 1) * (HD / 2); e0 += 32) {
    float v[2][16];
    tmem_ld16(trow + kOCol + e0, v[0]);
    tmem_ld16(trow + kOCol + e0 + 16, v[1]);
    tmem_ld_wait();
    if (qr < nq) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = head * HD + e0 + 8 * q;
        uint16_t* blk = p.o_act + ((size_t)(m >> 7) * (K >> 6) + (col >> 6)) * (kBM * 64);
        const int r = m & 127;
        const float* x = &v[q >> 1][(q & 1) * 8];
        *reinterpret_cast<uint4*>(blk + r * 64 + ((((col & 63) >> 3) ^ (r & 7)) << 3)) =
            make_uint4(pk_bf16(x[0] * inv, x[1] * inv), pk_bf16(x[2] * inv, x[3] * inv),
                       pk_bf16(x[4] * inv, x[5] * inv), pk_bf16(x[6] * inv, x[7] * inv));
      }
    }
  }
  if (!ok) atomicOr(p.err, 1u << 12);
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAtTmem);
  }
}

// The tensor-core kernel serves up to 3 x 128 keys per request (every score
// row in TMEM at once) and head dims 64 and 128; other shapes keep the
// mma.sync kernel.
bool battn_tc_supported(int S_max, int hd) {
  return S_max <= kAtMaxChunks * kAtChunk && (hd == 64 || hd == 128);
}

cudaError_t launch_battn_tc(const BAttnParams& p, cudaStream_t st) {
  const int qblocks = (p.Hq / p.Hkv * p.T + kAtRows - 1) / kAtRows;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.gridDim = dim3(qblocks, p.Hkv, p.B);
  cfg.blockDim = dim3(kAtThreads, 1, 1);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (p.hd == 128) {
    cfg.dynamicSmemBytes = AtCfg<128>::kSmem;
    cudaError_t e = cudaFuncSetAttribute(battn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)AtCfg<128>::kSmem);
    return e != cudaSuccess ? e : cudaLaunchKernelEx(&cfg, battn_tc_kernel<128>, p);
  }
  cfg.dynamicSmemBytes = AtCfg<64>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(battn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)AtCfg<64>::kSmem);
  return e != cudaSuccess ? e : cudaLaunchKernelEx(&cfg, battn_tc_kernel<64>, p);
}

}  // namespace fm
