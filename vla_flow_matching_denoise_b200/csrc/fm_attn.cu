// Batched GQA attention on the 5th-generation tensor cores ("LingBot-VLA on
// Thor (sm_110)", §3 FlashAttention-4: the denoise attention is grouped-query
// attention over the cached prefix keys and the chunk's own keys, pack_gqa).
//
// One CTA per (request b, KV group g, block of 128 query rows of that group:
// row (h % G) T + t for the group's G heads and the chunk's T tokens), four
// warps; thread i owns query row i (TMEM lane i of the M = 128 accumulators).
//   1. Thread 0 moves Q rows and, per 128-key chunk, K and V rows into shared
//      memory with one TMA copy per 64-element half of 128 rows (4-D views
//      (64 elements, half, row, segment) of the q buffer and the caches): both
//      store each row's 16-byte pieces swizzled by (row & 7), so every 128-byte
//      half row is already a row of the 128-byte-swizzled image tcgen05 reads,
//      and the copy lands as [half][128 rows][128 B].  K and V are
//      double-buffered and stream while the tensor cores work.
//   2. S = Q K^T for every chunk (up to 3 x 128 keys) accumulates in TMEM
//      columns [128 c, 128 c + 128) (K is the K-major B operand).
//   3. Each thread reads its S row twice: the row maximum, then
//      p = exp2(s log2(e) / sqrt(hd) - max) for valid keys (0 for the padding
//      keys of the last chunk), summing l in fp32 and storing p as bf16 into
//      the K-major image of P (over the Q and K buffers, which S has
//      finished with).  Every key is in TMEM at once, so the softmax is exact
//      in one pass and O is never rescaled.
//   4. O = P V accumulates in TMEM columns [384, 384 + hd); V rows, hd
//      contiguous, are the MN-major B operand as they arrive.
//   5. o = O / l in bf16 goes to the ACT128 activation of o_proj.
// Rows past the request's P_b + T (up to the cache's row count) hold finite
// values the kernels wrote earlier, rows past the cache are filled with zeros
// by the copy: their scores are masked and their probabilities are exactly 0.
// Query rows beyond G T stay in their own rows, which are not stored.
// Requests are independent and every sum runs in a fixed order
// (bit-reproducible).
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>

#include "fm_batch.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {

constexpr int kAtThreads = 128;
constexpr int kAtRows = 128;            // query rows per CTA (MMA M)
constexpr int kAtChunk = 128;           // keys per chunk (MMA N of S, K of O)
constexpr int kAtMaxChunks = 3;
constexpr int kAtTile = kAtRows * 128;  // bytes of one 128-row x 128-byte image
constexpr int kOCol = kAtMaxChunks * kAtChunk;   // first TMEM column of O

// Barriers: Q, K buffers (2), V buffers (2), S per chunk (3), O per chunk (3).
enum { BQ = 0, BK = 1, BV = 3, BS = 5, BO = 8, kAtBars = 11 };

template <int HD>
struct AtCfg {
  static constexpr int kHalves = HD / 64;                   // 128-byte halves of a row
  static constexpr int kImg = kHalves * kAtTile;            // Q / K / V image: [half][128 rows][128 B]
  static constexpr int kPBytes = 2 * kAtTile;               // P chunk: [key half][128 rows][128 B]
  // region A: Q, K0, K1 (later P of 3 chunks); region V: V0, V1
  static constexpr int kRegA = 3 * kImg > kAtMaxChunks * kPBytes ? 3 * kImg : kAtMaxChunks * kPBytes;
  static constexpr int kSmem = 1024 + kRegA + 2 * kImg + 256;
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
__global__ void __launch_bounds__(kAtThreads, 1) battn_tc_kernel(const __grid_constant__ BAttnParams p) {
  using C = AtCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = sm;                                    // region A
  uint8_t* kbuf[2] = {sm + C::kImg, sm + 2 * C::kImg};
  uint8_t* ps = sm;                                    // region A again, once S is complete
  uint8_t* vbuf[2] = {sm + C::kRegA, sm + C::kRegA + C::kImg};
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kRegA + 2 * C::kImg);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + kAtBars + 1);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int qb = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = p.Hq / p.Hkv, T = p.T;
  const int nq = G * T;                                // query rows of the group
  const long long budget = p.spin_budget;

  if (tid == 0) {
    for (int i = 0; i < kAtBars; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tslot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  grid_dep_wait();   // q and the chunk's cache rows come from the QKV GEMM

  const int S = p.P_dev[b] + T;                       // keys of this request
  const int nch = (S + kAtChunk - 1) / kAtChunk;
  bool ok = true;

  // 1: Q, the first two K chunks and the first two V chunks start streaming
  const int qseg = b * p.Hkv + g, kvseg = p.seg_base + qseg;
  if (tid == 0) {
    // K and V rows serve the group's other query blocks too: keep them in L2
    const uint64_t pol = policy_evict_first(), pol_kv = policy_evict_last();
    tma_tile<HD>(qs, &p.tm_q, qb * kAtRows, qseg, smem_u32(&bars[BQ]), pol);
    for (int c = 0; c < nch && c < 2; ++c) {
      tma_tile<HD>(kbuf[c], &p.tm_k, c * kAtChunk, kvseg, smem_u32(&bars[BK + c]), pol_kv);
      tma_tile<HD>(vbuf[c], &p.tm_v, c * kAtChunk, kvseg, smem_u32(&bars[BV + c]), pol_kv);
    }
  }
  __syncwarp();

  // 2: S = Q K^T per chunk (thread 32 issues); a third K chunk reuses buffer 0
  const uint32_t id_s = idesc_bf16(kAtRows, kAtChunk);
  if (tid == 32) {
    ok &= mbar_wait(smem_u32(&bars[BQ]), 0, budget);
    for (int c = 0; c < nch; ++c) {
      ok &= mbar_wait(smem_u32(&bars[BK + (c & 1)]), (uint32_t)(c >> 1), budget);
      tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < HD / 16; ++k16) {
        const uint32_t off = (uint32_t)((k16 >> 2) * kAtTile + (k16 & 3) * 32);
        mma_bf16(tmem + c * kAtChunk, desc_sw128(smem_u32(qs) + off), desc_sw128(smem_u32(kbuf[c & 1]) + off),
                 id_s, k16 > 0);
      }
      mma_commit(smem_u32(&bars[BS + c]));
    }
  }
  __syncwarp();
  if (tid == 0 && nch > 2) {
    ok &= mbar_wait(smem_u32(&bars[BS + 0]), 0, budget);
    tma_tile<HD>(kbuf[0], &p.tm_k, 2 * kAtChunk, kvseg, smem_u32(&bars[BK + 0]), policy_evict_last());
  }
  __syncwarp();
  // every S chunk complete: the last commit covers all earlier MMAs
  ok &= mbar_wait(smem_u32(&bars[BS + nch - 1]), 0, budget);
  tc_fence_after();

  // 3: softmax of row `tid` over the S keys; P over region A
  const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  float mx = -INFINITY;
  for (int c0 = 0; c0 < nch * kAtChunk; c0 += 32) {
    float v[2][16];
    tmem_ld16(trow + c0, v[0]);
    tmem_ld16(trow + c0 + 16, v[1]);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < S) mx = fmaxf(mx, v[j >> 4][j & 15]);
  }
  const float mb = mx * sl2;
  float l = 0.f;
  for (int c0 = 0; c0 < nch * kAtChunk; c0 += 32) {
    float v[2][16];
    tmem_ld16(trow + c0, v[0]);
    tmem_ld16(trow + c0 + 16, v[1]);
    tmem_ld_wait();
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const float s0 = v[(2 * j) >> 4][(2 * j) & 15], s1 = v[(2 * j + 1) >> 4][(2 * j + 1) & 15];
      const float e0 = c0 + 2 * j < S ? exp2f(fmaf(s0, sl2, -mb)) : 0.f;
      const float e1 = c0 + 2 * j + 1 < S ? exp2f(fmaf(s1, sl2, -mb)) : 0.f;
      l += e0;
      l += e1;
      pk[j] = pk_bf16(e0, e1);
    }
    // P chunk c0 / 128, key half (c0 % 128) / 64, pieces (c0 % 64) / 8 .. + 3
    const int c = c0 >> 7, kh = (c0 >> 6) & 1, pc0 = (c0 & 63) >> 3;
    uint8_t* row = ps + c * C::kPBytes + kh * kAtTile + tid * 128;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(row + (((pc0 + i) ^ (tid & 7)) << 4)) =
          make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // 4: O = P V per chunk (V: hd-contiguous rows = MN-major B); a third V
  // chunk reuses buffer 0 once the first chunk's MMAs are done
  const uint32_t id_o = idesc_bf16_bmn(kAtRows, HD);
  if (tid == 32) {
    tc_fence_after();
    for (int c = 0; c < nch; ++c) {
      ok &= mbar_wait(smem_u32(&bars[BV + (c & 1)]), (uint32_t)(c >> 1), budget);
      tc_fence_after();
#pragma unroll
      for (int k16 = 0; k16 < kAtChunk / 16; ++k16) {
        const uint32_t aoff = (uint32_t)((k16 >> 2) * kAtTile + (k16 & 3) * 32);
        mma_bf16(tmem + kOCol, desc_sw128(smem_u32(ps + c * C::kPBytes) + aoff),
                 desc_sw128_mn(smem_u32(vbuf[c & 1]) + (uint32_t)k16 * 2048u, kAtTile), id_o, (c | k16) != 0);
      }
      mma_commit(smem_u32(&bars[BO + c]));
    }
  }
  __syncwarp();
  if (tid == 0 && nch > 2) {
    ok &= mbar_wait(smem_u32(&bars[BO + 0]), 0, budget);
    tma_tile<HD>(vbuf[0], &p.tm_v, 2 * kAtChunk, kvseg, smem_u32(&bars[BV + 0]), policy_evict_last());
  }
  __syncwarp();
  ok &= mbar_wait(smem_u32(&bars[BO + nch - 1]), 0, budget);
  tc_fence_after();

  // 5: o = O / l -> ACT128 [Mp/128][Hq*hd/64] rows b T + t, columns h hd + e
  const int qr = qb * kAtRows + tid;
  const float inv = 1.0f / l;
  const int head = g * G + (qr < nq ? qr / T : 0), t = qr < nq ? qr % T : 0;
  const int m = b * T + t;
  const int K = p.Hq * HD;
  for (int e0 = 0; e0 < HD; e0 += 32) {
    float v[2][16];
    tmem_ld16(trow + kOCol + e0, v[0]);
    tmem_ld16(trow + kOCol + e0 + 16, v[1]);
    tmem_ld_wait();
    if (qr < nq) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = head * HD + e0 + 8 * i;
        uint16_t* blk = p.o_act + ((size_t)(m >> 7) * (K >> 6) + (col >> 6)) * (kBM * 64);
        const int r = m & 127;
        const float* x = &v[i >> 1][(i & 1) * 8];
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
    tmem_dealloc(tmem, 512);
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
