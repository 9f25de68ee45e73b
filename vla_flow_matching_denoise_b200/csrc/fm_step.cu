// Latency-mode denoise megakernel: one persistent launch runs
//   for each Euler step k:  in-proj;  L x (QKV+RoPE, GQA attention, o_proj +
//   gated residual, gate_up + SwiGLU, down + gated residual);  final
//   AdaRMSNorm + out-proj + Euler update
// for one 50-token action chunk ("LingBot-VLA on Thor (sm_110)", §1: a
// 36-layer expert with a per-step denoise loop; §2: fused AdaRMSNorm, SwiGLU
// tail, QKV+RoPE; §3: GQA denoise attention; "LingBot-VLA v2 Examples",
// CUDA Graph: the prefix KV cache is reused by every denoise step).
//
// Design (B200, one request):
//  * The grid is every co-resident cluster of 8 CTAs, one CTA per SM.  There
//    is no grid barrier: each phase's writers add 1 to that phase's counter
//    in global memory (release) once their outputs are stored, and a phase
//    waits (acquire, bounded spin) only for the counter of the outputs it
//    reads, right before it reads them; the polling thread then requests the
//    CTA's K-slice of the activations with one bulk copy.  Activations
//    alternate between two copies by layer parity.  Every wait of the compute
//    warps ends in a vote, so a wait that gives up sends them all the same way.
//  * Weights dominate the bytes (34.6 MB per layer at d = 1024), so warp 0 of
//    every CTA streams its share of every layer, in consumption order, through
//    a 126 KB shared-memory ring with 1-D bulk (TMA) copies, and requests the
//    next layer's span into L2 ahead of time.  The stream runs ahead across
//    phases, throttled by ring space and by at most two copies in flight (the
//    activation copies share the SM's bulk-copy engine).
//  * Each linear is split over clusters by output channels and, inside a
//    cluster, over its 8 CTAs by K and n-groups.  Warp 1 issues tcgen05.mma
//    with M = 64 token rows (50 valid + the shift row + padding), N = the
//    CTA's channels, accumulating fp32 in TMEM.
//  * Split-K partials leave TMEM through tcgen05.ld straight into registers
//    and go to the owner of each column with st.async into the owner's shared
//    memory, completing bytes on its mbarrier (a CTA's own slot with plain
//    shared stores); the owner reduces its KS slots in a fixed order (results
//    are bit-reproducible).  o_proj and down have the same owners, which keep
//    the residual stream h in registers across phases and layers.
//  * AdaRMSNorm is folded into the linears: the owner of a residual column
//    writes z = bf16(h (1 + s)) and, in row 50, the shift b; the consumer
//    linear's epilogue applies rstd(row) to rows 0..49 and adds row 50
//    (= b W^T).  This equals y W^T with y = h rstd (1 + s) + b.  Row sums of
//    h^2 are published per CTA and summed by the consumer in a fixed order.
//  * Attention (50 queries per head) runs per (KV group, block of 64 query
//    rows of that group's heads) on one cluster, keys split over its 8 CTAs,
//    mma.sync with an online softmax, partials pushed to the row owners for
//    the log-sum-exp combine.
//  * E4M3 / NVFP4 weights ("LingBot-VLA on Thor (sm_110)", §2: FP8 weight
//    path, FP4 gate_up) run in a second instantiation of the kernel with two
//    extra warps that widen the codes in the ring to the bf16 image (exact),
//    so the tensor cores still run bf16 x bf16; the per-output-row scale
//    multiplies the reduced fp32 sum in the epilogue.  The bf16 instantiation
//    carries none of that code.
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>
#include <type_traits>

#include "fm_internal.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {

// This CTA's share of one linear.
struct GemmView {
  int ng;        // channels of its n-group (0: idle cluster)
  int KS, ks, grp;
  int own;       // owned output columns
  int ownp;      // row stride (floats) of the staging / receive blocks, multiple of 4
  int nchunk;
  int base;      // first owned packed channel (gate_up: first owned u column)
  int pbase;     // index of the first owned column in the layer's scale table
  uint32_t recv_off;   // byte offset of the receive buffer in the work region
};

struct Ctrl {
  uint64_t full[kRingSlots];
  uint64_t empty[kRingSlots];
  uint64_t conv[kRingSlots];   // E4M3 weights: chunk widened to bf16
  uint64_t act_full;
  uint64_t mma_done;
  uint64_t recv;      // split-K / attention partials pushed by the cluster
  uint64_t att;       // attention tile loads
  uint64_t drain;
  uint64_t xsync;     // cluster rendezvous (8 arrivals)
  uint32_t ring_st[kRingSlots], ring_en[kRingSlots];   // producer only: chunk ranges in flight
  uint32_t tmem_slot;
  int abort;
  uint32_t writers[kNumFlags];       // CTAs that signal each hand-off per round
  alignas(16) float rstd[kRows];
  alignas(16) float red[8][kRows];   // written with float4 stores
  GemmView views[4];                 // this CTA's share of each linear (fixed per launch)
};
static_assert(offsetof(Ctrl, red) % 16 == 0 && offsetof(Ctrl, rstd) % 16 == 0, "vector alignment");

constexpr size_t kSmemBytes = 1024 + kRingBytes + kWorkBytes + ((sizeof(Ctrl) + 127) / 128) * 128;
static_assert(kSmemBytes <= (size_t)kSmemMax, "shared memory budget");

// Error codes (bit flags in p.err).
enum : uint32_t {
  E_FLAG = 1u << 0,
  E_RING_PROD = 1u << 1,
  E_RING_MMA = 1u << 2,
  E_RECV = 1u << 3,
  E_MMA_DONE = 1u << 4,
  E_ATT = 1u << 7,
  E_CONV = 1u << 8,
};

__device__ __forceinline__ bool wait_ab(uint32_t bar, uint32_t parity, long long budget,
                                        volatile int* abort) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test_sleep(bar, parity, 1000000u)) {
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

// Ring placement shared by producer and consumer: a chunk of `sz` bytes goes
// right after the previous one, or wraps to offset 0 when it does not fit.
__device__ __forceinline__ uint32_t ring_place(uint32_t& pos, uint32_t sz) {
  const uint32_t p = (pos + sz > (uint32_t)kRingBytes) ? 0u : pos;
  pos = p + sz;
  return p;
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}

// Element offset of (row r, column c) inside an ACT64 matrix.
__device__ __forceinline__ size_t act64_off(int r, int c) {
  return (size_t)(c >> 6) * (kRows * 64) + (size_t)r * 64 + ((((c & 63) >> 3) ^ (r & 7)) << 3) + (c & 7);
}

// Element index inside a row of hd bf16 values stored with 16-byte pieces
// swizzled by (row & 7).
__device__ __forceinline__ int swz(int row, int e) {
  return ((((e >> 3) ^ (row & 7))) << 3) | (e & 7);
}

__device__ __forceinline__ unsigned long long gtimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctx {
  const StepParams* p;
  uint8_t* work;
  Ctrl* ctl;
  uint32_t tmem;
  int cta, cluster, rank;
  int tid;              // 0..127 within the compute warps
  int warp;             // 2..5
  int lane;
  uint32_t gemm_count;  // GEMM phases run (parity of act_full / mma_done)
  uint32_t recv_count, att_count, xs_count;
  uint32_t phase;       // phases passed (profiling marks)
  uint32_t ep[kNumFlags];   // hand-off rounds signalled so far, per counter
  float2 hres[4];           // this thread's owned residual values (o_proj and down share owners)
  int P;                // prefix length (read from the device)
  bool ok;
};

__device__ __forceinline__ void compute_sync() { named_bar_sync(1, kComputeWarps * 32); }

// Every compute thread passes its view of the phase's health (its own waits
// and the CTA's abort flag); all leave with the same answer, so a wait that
// gave up on one thread sends every thread the same way and none is left
// waiting at a later barrier.
__device__ __forceinline__ bool compute_vote(const Ctx& c, bool ok) {
  ok = ok && *(volatile int*)&c.ctl->abort == 0;
  return named_bar_and(1, kComputeWarps * 32, ok);
}

// Phase timeline (profiling only): mark `slot` of the current phase: 0 start,
// 1 MMA / attention compute done, 2 partials pushed, 3 partials received,
// 4 epilogue done, 5 barrier arrival issued, 6 partials staged, 7 staging
// synchronised, 8.. phase-specific points.
__device__ __forceinline__ void tmark(const Ctx& c, int slot) {
  if (c.p->tlog != nullptr && c.tid == 0) {
    const int idx = (int)c.phase * 16 + slot;
    if (idx < c.p->tlog_mma_off) c.p->tlog[(size_t)c.cta * c.p->tlog_stride + idx] = gtimer();
  }
}

__device__ __forceinline__ void fail(Ctx& c, uint32_t code) {
  atomicOr(c.p->err, code);
  c.ctl->abort = 1;
  c.ok = false;
}

// Bulk loads of `nch` 8 KB activation blocks (one thread), completing on act_full.
__device__ __forceinline__ void issue_act(const Ctx& c, const uint16_t* src, int nch) {
  const uint64_t pol = policy_evict_last();
  const uint32_t bar = smem_u32(&c.ctl->act_full);
  // the K-slice's blocks are consecutive in the ACT64 layout and in the work
  // region: one copy (fewer requests queued behind the weight stream's)
  mbar_arrive_expect_tx(bar, (uint32_t)nch * 8192u);
  bulk_g2s(smem_u32(c.work), src, (uint32_t)nch * 8192u, bar, pol);
}

// Waits until hand-off counter f has seen every writer of every round
// signalled so far (one thread polls, bounded), makes the data visible to
// this CTA's bulk copies and releases the compute warps.  A GEMM phase passes
// its K-slice of the activations (`act`, `nch` blocks), which the polling
// thread requests at once, before the other threads are released.
__device__ __forceinline__ void wait_flag(Ctx& c, int f, const uint16_t* act = nullptr, int nch = 0) {
  if (!c.ok) return;
  const uint32_t target = c.ep[f] * c.ctl->writers[f];
  if (c.tid == 0) {
    if (target > 0u) {
      const uint32_t* cnt = c.p->flags + f * kFlagStride;
      const long long t0 = clock64();
      uint32_t it = 0;
      while (ld_acquire_u32(cnt) < target) {
        if ((++it & 15u) == 0u &&
            (*(volatile uint32_t*)c.p->err != 0u || clock64() - t0 > c.p->spin_budget)) {
          fail(c, E_FLAG);
          break;
        }
      }
      fence_proxy_async_global();
    }
    if (act != nullptr && c.ok) issue_act(c, act, nch);
  }
  c.ok = compute_vote(c, c.ok);
  tmark(c, 0);
}

// Ends a phase: a writer CTA orders its stores (generic and async proxy)
// before one release add on counter f; every CTA counts the round.
__device__ __forceinline__ void signal(Ctx& c, int f, bool wrote) {
  if (c.ok && wrote) {
    tmark(c, 4);
    fence_proxy_async_global();
    tmark(c, 13);
    compute_sync();
    tmark(c, 14);
    if (c.tid == 0) red_release_add(c.p->flags + f * kFlagStride, 1u);
    tmark(c, 5);
  }
  ++c.ep[f];
  ++c.phase;
}

// ------------------------------------------------------------ producer warp
__device__ __noinline__ void producer(const StepParams& p, uint8_t* ring, Ctrl* ctl, int cta, int cluster) {
  const uint64_t pol = policy_evict_first();
  uint32_t nch[4], bytes[4];
  for (int g = 0; g < 4; ++g) {
    const int ng = p.g[g].ng[cluster];
    nch[g] = ng > 0 ? (uint32_t)p.g[g].nchunk : 0u;
    bytes[g] = (uint32_t)ng * 128u;
  }
  // E4M3 / NVFP4: a chunk's codes land at the end of its slot and are
  // widened in place; copy bytes per chunk row: 128 (bf16), 64, 36
  uint32_t rowb[4];
  for (int g = 0; g < 4; ++g) rowb[g] = p.wfmt[g] == 0 ? 128u : p.wfmt[g] == 1 ? 64u : 36u;
  // byte range of every chunk in flight, by barrier slot: in shared memory
  // (a local array indexed at run time lives in local memory, whose L1
  // share is small next to 227 KB of shared memory: every scan of the ring
  // then waited on L2)
  uint32_t* const st = ctl->ring_st;
  uint32_t* const en = ctl->ring_en;
  uint32_t head = 0, tail = 0, pos = 0;
  const uint32_t span0 = p.span_off[cta];
  // this CTA's bytes of one layer (one contiguous span per layer)
  uint32_t span = 0;
  for (int g = 0; g < 4; ++g) span += nch[g] * (bytes[g] >> 7) * rowb[g];
  // The ring holds less than one layer of this CTA's weights (gate_up alone
  // can exceed it), so the span of the layer after the one being streamed is
  // requested into L2 ahead of time: ring refills inside a phase then come
  // from L2 instead of waiting on HBM.
  auto prefetch_layer = [&](int l) {
    const uint8_t* a = p.arena + (size_t)l * p.layer_bytes + span0;
    for (uint32_t o = 0; o < span; o += 65536u) bulk_prefetch_l2(a + o, min(65536u, span - o));
  };
  if (span > 0) prefetch_layer(p.layer0);
  bool good = true;
  for (int s = p.step0; s < p.step1 && good; ++s) {
    for (int l = p.layer0; l < p.layer1 && good; ++l) {
      if (span > 0 && (l + 1 < p.layer1 || s + 1 < p.step1)) prefetch_layer(l + 1 < p.layer1 ? l + 1 : p.layer0);
      const uint8_t* src = p.arena + (size_t)l * p.layer_bytes + span0;
      for (int g = 0; g < 4 && good; ++g) {
        for (uint32_t i = 0; i < nch[g]; ++i) {
          const uint32_t sz = bytes[g];
          const uint32_t at = ring_place(pos, sz);
          // Wait until no chunk still in flight overlaps [at, at + sz) and a
          // barrier slot is free.
          for (;;) {
            bool conflict = head - tail >= (uint32_t)kRingSlots;
            for (uint32_t q = tail; !conflict && q < head; ++q) {
              const uint32_t a = st[q % kRingSlots], b = en[q % kRingSlots];
              if (a < at + sz && at < b) conflict = true;
            }
            if (!conflict) break;
            if (!wait_ab(smem_u32(&ctl->empty[tail % kRingSlots]), (tail / kRingSlots) & 1,
                         p.spin_budget, &ctl->abort)) {
              good = false;
              break;
            }
            ++tail;
          }
          if (!good) break;
          const uint32_t slot = head % kRingSlots;
          st[slot] = at;
          en[slot] = at + sz;
          if (p.tlog != nullptr && (int)head < p.tlog_chunks)
            p.tlog[(size_t)cta * p.tlog_stride + p.tlog_chunk_off + p.tlog_chunks + head] = gtimer();
          const uint32_t csz = (sz >> 7) * rowb[g];
          // at most 2 weight copies in flight: a phase's activation copy shares
          // this SM's bulk-copy engine and must not queue behind a deep stream
          if (head >= 2u) {
            const uint32_t q = head - 2u;
            if (!wait_ab(smem_u32(&ctl->full[q % kRingSlots]), (q / kRingSlots) & 1, p.spin_budget, &ctl->abort)) {
              good = false;
              break;
            }
          }
          mbar_arrive_expect_tx(smem_u32(&ctl->full[slot]), csz);
          bulk_g2s(smem_u32(ring + at + (sz - csz)), src, csz, smem_u32(&ctl->full[slot]), pol);
          src += csz;
          ++head;
        }
      }
    }
  }
  if (!good && !ctl->abort) {
    atomicOr(p.err, E_RING_PROD);
    ctl->abort = 1;
  }
  // Every issued copy must land before the CTA exits.
  for (uint32_t q = tail; q < head; ++q)
    mbar_wait(smem_u32(&ctl->full[q % kRingSlots]), (q / kRingSlots) & 1, p.spin_budget);
}

// ------------------------------------------------------------ widening warps
// E4M3 -> bf16, in place: chunk rows of 64 codes sit in the upper half of the
// slot; row r becomes the 128-byte swizzled bf16 row r.  Every thread loads
// all of its pieces before any thread stores (named barrier), so no store can
// overwrite codes not yet read.  ctid: 0 .. 32 * kConvWarps - 1.
__device__ __noinline__ void converter(const StepParams& p, uint8_t* ring, Ctrl* ctl, int cluster, int ctid) {
  constexpr int kCT = 32 * kConvWarps;
  constexpr int kMaxPieces = 256 * 4 / kCT;   // 16-byte code pieces per thread (ng <= 256)
  uint32_t nch[4], bytes[4];
  for (int g = 0; g < 4; ++g) {
    const int ng = p.g[g].ng[cluster];
    nch[g] = ng > 0 ? (uint32_t)p.g[g].nchunk : 0u;
    bytes[g] = (uint32_t)ng * 128u;
  }
  uint32_t it = 0, pos = 0;
  bool good = true;
  for (int s = p.step0; s < p.step1 && good; ++s) {
    for (int l = p.layer0; l < p.layer1 && good; ++l) {
      for (int g = 0; g < 4 && good; ++g) {
        const int npieces = (int)(bytes[g] >> 5);   // E4M3: ng rows x 4 pieces
        for (uint32_t c = 0; c < nch[g]; ++c, ++it) {
          const uint32_t at = ring_place(pos, bytes[g]);
          const uint32_t slot = it % kRingSlots;
          if (p.wfmt[g] == 0) continue;   // bf16 chunk: the MMA warp waits on `full` itself
          if (!wait_ab(smem_u32(&ctl->full[slot]), (it / kRingSlots) & 1, p.spin_budget, &ctl->abort)) {
            good = false;
            break;
          }
          uint8_t* base = ring + at;
          if (p.wfmt[g] == 1) {
            const uint8_t* codes = base + (bytes[g] >> 1);
            uint4 v[kMaxPieces];
#pragma unroll
            for (int j = 0; j < kMaxPieces; ++j) {
              const int i = ctid + kCT * j;
              if (i < npieces) v[j] = *reinterpret_cast<const uint4*>(codes + 16 * i);
            }
            named_bar_sync(2, kCT);
#pragma unroll
            for (int j = 0; j < kMaxPieces; ++j) {
              const int i = ctid + kCT * j;
              if (i >= npieces) break;
              const int r = i >> 2, q = i & 3;   // row, 16-code quarter -> bf16 pieces 2q, 2q + 1
              const uint32_t w[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
              uint32_t o[8];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                o[2 * k] = e4m3x2_to_bf16x2((uint16_t)(w[k] & 0xFFFFu));
                o[2 * k + 1] = e4m3x2_to_bf16x2((uint16_t)(w[k] >> 16));
              }
              uint8_t* row = base + (r >> 3) * 1024 + (r & 7) * 128;
              *reinterpret_cast<uint4*>(row + (((2 * q) ^ (r & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
              *reinterpret_cast<uint4*>(row + (((2 * q + 1) ^ (r & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
          } else {
            // NVFP4 rows: 32 bytes of E2M1 codes (two per byte, first in the low
            // nibble), then 4 E4M3 scales, one per 16-column block; every code x
            // scale product is exact in f16 and in bf16
            constexpr int kMaxRows = 256 / kCT;
            const int R = (int)(bytes[g] >> 7);
            const uint8_t* src = base + bytes[g] - (uint32_t)R * 36u;
            uint4 c0[kMaxRows], c1[kMaxRows];
            uint32_t scw[kMaxRows];
#pragma unroll
            for (int j = 0; j < kMaxRows; ++j) {
              const int q = ctid + kCT * j;
              if (q < R) {
                c0[j] = *reinterpret_cast<const uint4*>(src + 32 * q);
                c1[j] = *reinterpret_cast<const uint4*>(src + 32 * q + 16);
                scw[j] = *reinterpret_cast<const uint32_t*>(src + 32 * R + 4 * q);
              }
            }
            named_bar_sync(2, kCT);
#pragma unroll
            for (int j = 0; j < kMaxRows; ++j) {
              const int q = ctid + kCT * j;
              if (q >= R) break;
              const uint32_t cw[8] = {c0[j].x, c0[j].y, c0[j].z, c0[j].w, c1[j].x, c1[j].y, c1[j].z, c1[j].w};
              uint8_t* row = base + (q >> 3) * 1024 + (q & 7) * 128;
#pragma unroll
              for (int b = 0; b < 4; ++b) {
                const uint32_t s2 = e4m3_to_f16x2_bcast(scw[j] >> (8 * b));
                uint32_t o[8];
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  o[k] = f16x2_mul_to_bf16x2(e2m1x2_to_f16x2((cw[2 * b + (k >> 2)] >> (8 * (k & 3))) & 0xFFu), s2);
                *reinterpret_cast<uint4*>(row + (((2 * b) ^ (q & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(row + (((2 * b + 1) ^ (q & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
              }
            }
          }
          // generic-proxy stores must be visible to the tensor cores' reads
          fence_proxy_async_smem();
          mbar_arrive(smem_u32(&ctl->conv[slot]));
        }
      }
    }
  }
  if (!good && !ctl->abort) {
    atomicOr(p.err, E_CONV);
    ctl->abort = 1;
  }
}

// ------------------------------------------------------------ MMA warp
__device__ __noinline__ void mma_issuer(const StepParams& p, uint8_t* ring, uint8_t* work, Ctrl* ctl,
                           uint32_t tmem, int cluster) {
  // per-linear values in registers: the linear loop below is unrolled
  uint32_t nch[4], bytes[4], idesc[4], wide[4];
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const int ng = p.g[g].ng[cluster];
    nch[g] = ng > 0 ? (uint32_t)p.g[g].nchunk : 0u;
    bytes[g] = (uint32_t)ng * 128u;
    idesc[g] = idesc_bf16(kRows, ng > 0 ? ng : 16);
    wide[g] = p.wfmt[g] != 0 ? 1u : 0u;
  }
  unsigned long long* const tlog = p.tlog;
  const int tlog_row = p.tlog_stride * (int)blockIdx.x, tlog_mma = p.tlog_mma_off, tlog_chunk = p.tlog_chunk_off,
            tlog_chunks = p.tlog_chunks, tlog_stride = p.tlog_stride;
  const long long budget = p.spin_budget;
  uint32_t it = 0, pos = 0, gemm_count = 0;
  bool good = true;
  const uint32_t a_base = smem_u32(work);
  const uint32_t r_base = smem_u32(ring);
  for (int s = p.step0; s < p.step1 && good; ++s) {
    for (int l = p.layer0; l < p.layer1 && good; ++l) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        if (!good || nch[g] == 0) continue;
        if (!wait_ab(smem_u32(&ctl->act_full), gemm_count & 1, budget, &ctl->abort)) {
          good = false;
          continue;
        }
        tc_fence_after();
        if (tlog != nullptr && tlog_mma + 2 * (int)gemm_count < tlog_stride)
          tlog[tlog_row + tlog_mma + 2 * (int)gemm_count] = gtimer();
#pragma unroll 1
        for (uint32_t c = 0; c < nch[g]; ++c, ++it) {
          const uint32_t at = ring_place(pos, bytes[g]);
          const uint32_t slot = it % kRingSlots;
          if (!wait_ab(smem_u32(wide[g] ? &ctl->conv[slot] : &ctl->full[slot]), (it / kRingSlots) & 1, budget,
                       &ctl->abort)) {
            good = false;
            break;
          }
          if (tlog != nullptr && (int)it < tlog_chunks) tlog[tlog_row + tlog_chunk + it] = gtimer();
          tc_fence_after();
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_bf16(tmem, desc_sw128(a_base + c * 8192 + k16 * 32),
                     desc_sw128(r_base + at + k16 * 32), idesc[g], (c | k16) != 0);
          mma_commit(smem_u32(&ctl->empty[slot]));
        }
        if (!good) continue;
        if (tlog != nullptr && tlog_mma + 2 * (int)gemm_count + 1 < tlog_stride)
          tlog[tlog_row + tlog_mma + 2 * (int)gemm_count + 1] = gtimer();
        mma_commit(smem_u32(&ctl->mma_done));
        ++gemm_count;
      }
    }
  }
  if (!good && !ctl->abort) {
    atomicOr(p.err, E_RING_MMA);
    ctl->abort = 1;
  }
  // Drain: all issued MMAs must finish before TMEM is released.
  mma_commit(smem_u32(&ctl->drain));
  mbar_wait(smem_u32(&ctl->drain), 0, budget);
}

// ------------------------------------------------------------ compute warps
__device__ __forceinline__ const float* mod_vec(const StepParams& p, int step, int l, int which) {
  return p.mod + (size_t)step * p.n_mod + ((size_t)6 * l + which) * p.d;
}

constexpr int kMaxPairs = 4;    // owned column pairs per residual thread (checked by the planner)
constexpr int kAuxBytes = 8 * 1024;   // end of the work region: per-thread epilogue operands
constexpr int kAuxRows = kAuxBytes / (128 * 8);   // float2 rows per compute thread

// Computed once per launch into shared memory (make_views); the phases read
// it from there instead of re-deriving it from the launch parameters.
__device__ GemmView compute_view(const StepParams& p, int g, int cluster, int rank) {
  const GemmPlan& gp = p.g[g];
  GemmView v;
  v.ng = gp.ng[cluster];
  v.KS = gp.KS;
  v.ks = rank % gp.KS;
  v.grp = rank / gp.KS;
  v.own = v.ng / gp.KS;
  v.ownp = (v.own + 3) & ~3;
  v.nchunk = gp.nchunk;
  v.base = (g == G_GU) ? gp.ch_off[cluster] + v.grp * (v.ng / 2) + v.ks * (v.own / 2)
                       : gp.ch_off[cluster] + v.grp * v.ng + v.ks * v.own;
  v.pbase = (g == G_GU) ? 2 * gp.ch_off[cluster] + v.grp * v.ng + v.ks * v.own : v.base;
  const uint32_t a_bytes = (uint32_t)v.nchunk * 8192u;
  const uint32_t s_bytes = (uint32_t)(v.KS * kRecvRows * v.ownp * 4);
  v.recv_off = ((a_bytes > s_bytes ? a_bytes : s_bytes) + 15u) & ~15u;
  return v;
}

__device__ __forceinline__ GemmView gemm_view(const Ctx& c, int g) { return c.ctl->views[g]; }

// Row scales of two adjacent owned columns (E4M3 weights); 1 for bf16, where
// the product is exact and leaves the result unchanged.
__device__ __forceinline__ float2 wscale2(const Ctx& c, int g, int l, int idx) {
  const StepParams& p = *c.p;
  if (p.wscale == nullptr) return make_float2(1.f, 1.f);
  return *reinterpret_cast<const float2*>(p.wscale + (size_t)l * p.sc_stride + p.sc_off[g] + idx);
}

// Arms the receive barrier for the split-K partials the cluster will push
// here in GEMM g (safe before the input is ready: a peer pushes only after
// its own input wait, which this CTA's previous phase has released).
__device__ __forceinline__ void arm_recv(const Ctx& c, const GemmView& v) {
  // this CTA's own slot is written with plain shared-memory stores
  if (c.tid == 0)
    mbar_arrive_expect_tx(smem_u32(&c.ctl->recv), (uint32_t)((v.KS - 1) * kRecvRows * v.own * 4));
}

// Waits for the MMAs and sends rows 0..50 of the fp32 partial sums to the
// owners of their columns.  With the M = 64 accumulator, rows 16 q .. 16 q +
// 15 sit in TMEM lanes 32 q .. 32 q + 15 of warp quarter q; a 16x256b load
// gives lane t rows 16 q + t/4 and + 8 and column pairs 2 (t % 4) + 8 j.  One
// exchange between lanes t and t ^ 1 leaves every lane four consecutive
// columns of one row (even lanes the low row, odd lanes the high row), which
// go to the column's owner as one 16-byte st.async into its receive slot
// `ks`, completing bytes on the owner's receive barrier.  Owners hold a
// multiple of 4 columns, so a piece never straddles two owners.
__device__ __forceinline__ void push_send(Ctx& c, const GemmView& v) {
  if (!c.ok) return;
  Ctrl* const ctl = c.ctl;
  tmark(c, 12);
  if (!wait_ab(smem_u32(&ctl->mma_done), c.gemm_count & 1, c.p->spin_budget, &ctl->abort)) {
    fail(c, E_MMA_DONE);
    return;
  }
  ++c.gemm_count;
  tc_fence_after();
  tmark(c, 1);
  const int q = c.warp & 3, lane = c.lane;
  const bool odd = (lane & 1) != 0;
  const int r = 16 * q + (lane >> 2) + (odd ? 8 : 0);
  const bool act = r < kRecvRows;
  const uint32_t tb = c.tmem + ((uint32_t)(32 * q) << 16);
  const int ng = v.ng, own = v.own;
  const uint32_t recv_local = smem_u32(c.work + v.recv_off), bar_local = smem_u32(&ctl->recv);
  const uint32_t row_bytes = (uint32_t)((v.ks * kRecvRows + r) * v.ownp) * 4u;
  const int rank0 = v.grp * v.KS;
  // owner and column inside it of this lane's first column (2 (lane & 2)),
  // advanced by 8 columns per piece
  int o = 0, lc = 2 * (lane & 2);
  while (lc >= own) {
    lc -= own;
    ++o;
  }
#pragma unroll 1
  for (int c0 = 0; c0 < ng; c0 += 32) {
    float x[16];
    tmem_ld_16x256b_x4(tb + c0, x);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float sa = odd ? x[4 * j] : x[4 * j + 2];
      const float sb = odd ? x[4 * j + 1] : x[4 * j + 3];
      const float ra = __shfl_xor_sync(0xffffffffu, sa, 1);
      const float rb = __shfl_xor_sync(0xffffffffu, sb, 1);
      if (act && c0 + 8 * j < ng) {
        const uint32_t rk = (uint32_t)(rank0 + o);
        const float e0 = odd ? ra : x[4 * j], e1 = odd ? rb : x[4 * j + 1];
        const float e2 = odd ? x[4 * j + 2] : ra, e3 = odd ? x[4 * j + 3] : rb;
        if (rk == (uint32_t)c.rank) {
          st_shared_v4(recv_local + row_bytes + 4u * lc, e0, e1, e2, e3);
        } else {
          const uint32_t dst = map_shared_rank(recv_local, rk) + row_bytes + 4u * lc;
          st_async_v4(dst, e0, e1, e2, e3, map_shared_rank(bar_local, rk));
        }
      }
      lc += 8;
      while (lc >= own) {
        lc -= own;
        ++o;
      }
    }
  }
  tc_fence_before();
  tmark(c, 2);
}

// Every compute thread waits for the peers' partials, then all meet (this
// CTA's own slot was stored by all of them) and agree on the outcome, so a
// wait that gives up sends every thread the same way.
__device__ __forceinline__ void push_wait(Ctx& c) {
  bool w = c.ok && wait_ab(smem_u32(&c.ctl->recv), c.recv_count & 1, c.p->spin_budget, &c.ctl->abort);
  w = compute_vote(c, w);
  if (!w) {
    if (c.ok) fail(c, E_RECV);
    c.ok = false;
    return;
  }
  ++c.recv_count;
  tmark(c, 3);
}

// rstd[t] = (sum over CTAs of the partial sums of h^2 / d + eps)^-1/2.
// Thread tid adds rows 4*(tid%16)..+3 of CTAs tid/16 + 8k (independent float4
// loads, four per round); the eight groups are then added in a fixed order.
__device__ __forceinline__ void load_rstd(const Ctx& c, const float* sumsq) {
  const int T = c.p->T, n = c.p->n_ctas, d = c.p->d;
  const float eps = c.p->eps;
  const int tid = c.tid;
  Ctrl* const ctl = c.ctl;
  const float4* src = reinterpret_cast<const float4*>(sumsq);
  const int nf4 = n * (kRows / 4);
  // every load in flight at once (one L2 round trip), then added in CTA order
  constexpr int kMaxF = kMaxClusters * kClusterSize * (kRows / 4) / 128;
  float4 x[kMaxF];
#pragma unroll
  for (int j = 0; j < kMaxF; ++j) {
    const int f = tid + 128 * j;
    x[j] = f < nf4 ? src[f] : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int j = 0; j < kMaxF; ++j) {
    a.x += x[j].x; a.y += x[j].y; a.z += x[j].z; a.w += x[j].w;
  }
  *reinterpret_cast<float4*>(&ctl->red[tid >> 4][4 * (tid & 15)]) = a;
  compute_sync();
  if (tid < T) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) s += ctl->red[g][tid];
    ctl->rstd[tid] = 1.0f / sqrtf(s / (float)d + eps);
  }
}

// Sum over the KS senders of two adjacent received columns of row r.
__device__ __forceinline__ float2 recv_sum2(const float* rb, int KS, int ownp, int r, int lc) {
  // every slot's load in flight at once, then the sum in slot order
  const float* p0 = rb + r * ownp + lc;
  const int stride = kRecvRows * ownp;
  float2 x[kClusterSize];
#pragma unroll
  for (int s = 0; s < kClusterSize; ++s)
    x[s] = s < KS ? *reinterpret_cast<const float2*>(p0 + s * stride) : make_float2(0.f, 0.f);
  float2 a = x[0];
#pragma unroll
  for (int s = 1; s < kClusterSize; ++s) {
    a.x += x[s].x;
    a.y += x[s].y;
  }
  return a;
}

// As recv_sum2 for exactly N senders: no predicated slots (the epilogues call
// it when the plan's KS equals N; same slot order, same sum).
template <int N>
__device__ __forceinline__ float2 recv_sum2n(const float* rb, int ownp, int r, int lc) {
  const float* p0 = rb + r * ownp + lc;
  const int stride = kRecvRows * ownp;
  float2 x[N];
#pragma unroll
  for (int s = 0; s < N; ++s) x[s] = *reinterpret_cast<const float2*>(p0 + s * stride);
  float2 a = x[0];
#pragma unroll
  for (int s = 1; s < N; ++s) {
    a.x += x[s].x;
    a.y += x[s].y;
  }
  return a;
}

// Fixed item assignment of the epilogues: thread tid takes column pair
// tid % npair for rows tid / npair + k * (128 / npair).
struct PairRows {
  int pr, t0, dt;
  bool active;
};
__device__ __forceinline__ PairRows pair_rows(int tid, int npair) {
  PairRows r;
  const int per = 128 / npair;
  r.pr = tid % npair;
  r.t0 = tid / npair;
  r.dt = per;
  r.active = npair > 0 && tid < per * npair;
  return r;
}

// QKV: reduce, rstd + shift row, RoPE -> q buffer and the chunk rows of the
// KV cache.
__device__ __forceinline__ void phase_qkv(Ctx& c, int step, int l) {
  if (!c.ok) return;
  const StepParams& p = *c.p;
  const GemmView v = gemm_view(c, G_QKV);
  if (v.ng == 0) return;
  arm_recv(c, v);
  const int T = p.T, hd = p.hd, half = hd / 2, G = p.Hq / p.Hkv;
  const int qn = p.Hq * hd, kn = p.Hkv * hd, N = p.g[G_QKV].N;
  const int P = c.P;
  const PairRows pa = pair_rows(c.tid, v.own / 2);
  const int n = v.base + 2 * pa.pr;
  const bool act = pa.active && n < N;
  // destination of this thread's column pair: q (kind 0), k (1) or v (2)
  const int kind = n < qn ? 0 : n < qn + kn ? 1 : 2;
  const int nn = kind == 0 ? n : kind == 1 ? n - qn : n - qn - kn;
  const int head = nn / hd, w = nn % hd, ri = w >> 1;
  uint16_t* dst;
  int row_off;    // row index of token 0
  if (kind == 0) {
    dst = p.qbuf + (size_t)(head / G) * p.q_rows * hd;
    row_off = (head % G) * T;
  } else {
    dst = (kind == 1 ? p.kcache : p.vcache) + (((size_t)l * p.B_cap + p.b) * p.Hkv + head) * p.S_max * hd;
    row_off = P;
  }
  // stage the rotation of every row of this thread before the input is
  // ready (all loads at once; the planner keeps the rows per thread within
  // kAuxRows)
  float2* aux = reinterpret_cast<float2*>(c.work + kWorkBytes - kAuxBytes) + c.tid;
  if (act && kind < 2) {
    const float2* rope = reinterpret_cast<const float2*>(p.rope) + (size_t)p.b * T * half + ri;
    float2 rv[kAuxRows];
#pragma unroll
    for (int k = 0; k < kAuxRows; ++k) {
      const int t = pa.t0 + k * pa.dt;
      if (t < T) rv[k] = rope[t * half];
    }
#pragma unroll
    for (int k = 0; k < kAuxRows; ++k)
      if (pa.t0 + k * pa.dt < T) aux[k * 128] = rv[k];
  }
  wait_flag(c, F_Z, p.z_a + (size_t)(l & 1) * kRows * p.d + (size_t)(v.ks * v.nchunk) * (kRows * 64), v.nchunk);
  tmark(c, 11);
  load_rstd(c, p.sumsq_a);
  const float2 sc = act ? wscale2(c, G_QKV, l, v.pbase + 2 * pa.pr) : make_float2(1.f, 1.f);
  push_send(c, v);
  push_wait(c);
  if (!c.ok || !act) return;
  const float* rb = reinterpret_cast<const float*>(c.work + v.recv_off);
  const float* rstd = c.ctl->rstd;
  const float2 bsh = recv_sum2(rb, v.KS, v.ownp, kBiasRow, 2 * pa.pr);
  tmark(c, 8);
  // the row loop is instruction-bound (one compute warp per scheduler): the
  // plan's split (four ways) gets a copy without predicated receive slots
  auto rows = [&](auto ksn) {
    constexpr int N = decltype(ksn)::value;
#pragma unroll 1
    for (int t = pa.t0, k = 0; t < T; t += pa.dt, ++k) {
      const float2 a = N > 0 ? recv_sum2n<(N > 0 ? N : 1)>(rb, v.ownp, t, 2 * pa.pr)
                             : recv_sum2(rb, v.KS, v.ownp, t, 2 * pa.pr);
      const float rs = rstd[t];
      const float y0 = fmaf(rs, a.x, bsh.x) * sc.x, y1 = fmaf(rs, a.y, bsh.y) * sc.y;
      const int rr = row_off + t;
      uint16_t* rowp = dst + (size_t)rr * hd;
      if (kind < 2) {
        const float2 r = aux[k * 128];
        rowp[swz(rr, ri)] = bf16_bits(y0 * r.x - y1 * r.y);
        rowp[swz(rr, ri + half)] = bf16_bits(y1 * r.x + y0 * r.y);
      } else {
        *reinterpret_cast<uint32_t*>(rowp + swz(rr, w)) = pack_bf16(y0, y1);
      }
    }
  };
  if (v.KS == 4) rows(std::integral_constant<int, 4>{});
  else rows(std::integral_constant<int, 0>{});
}

// Attention for one (KV group, 64-row block of the group's G*T query rows);
// this CTA takes one key range of [prefix ; chunk].
template <int HD>
__device__ __forceinline__ void attention_unit(Ctx& c, int l, int grp, int blk) {
  const StepParams& p = *c.p;
  constexpr int KSTEPS = HD / 16;
  constexpr int DT = HD / 8;         // n-tiles of the output
  constexpr int RWP = HD + 4;        // floats per pushed row: o, m, l, padding
  const int G = p.Hq / p.Hkv;
  const int T = p.T;
  const int S = c.P + T;
  const int kpc = ((S + kClusterSize * 16 - 1) / (kClusterSize * 16)) * 16;
  const int rank = c.rank, tid = c.tid, lane = c.lane;
  const int k0 = rank * kpc;
  const int k1 = min(S, k0 + kpc);
  const int row0 = blk * 64;                       // first query row of the block
  const int nrows = min(64, G * T - row0);
  const long long budget = p.spin_budget;
  Ctrl* const ctl = c.ctl;
  uint8_t* const qs = c.work;
  uint8_t* const ks_ = c.work + 64 * HD * 2;
  uint8_t* const vs_ = ks_ + 64 * HD * 2;
  float* const rb = reinterpret_cast<float*>(vs_ + 64 * HD * 2);    // [8 senders][8 rows][RWP]
  float* const stg = reinterpret_cast<float*>(c.work);              // [64 rows][RWP], after compute
  const uint32_t qa = smem_u32(qs), ka = smem_u32(ks_), va = smem_u32(vs_);
  const uint32_t att_bar = smem_u32(&ctl->att);
  const uint64_t pol = policy_evict_last();
  const size_t kvoff = ((((size_t)l * p.B_cap + p.b) * p.Hkv + grp) * p.S_max) * HD;
  const uint16_t* kg = p.kcache + kvoff;
  const uint16_t* vg = p.vcache + kvoff;
  const uint16_t* qg = p.qbuf + ((size_t)grp * p.q_rows + row0) * HD;
  if (tid == 0) {
    // every CTA of the cluster sends 8 rows to each owner
    mbar_arrive_expect_tx(smem_u32(&ctl->recv), (uint32_t)(kClusterSize * 8 * RWP * 4));
  }

  const int w4 = c.warp - 2;               // rows 16*w4 .. +15
  const int r0 = 16 * w4;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  // ldmatrix lane addresses (row-swizzled 16-byte pieces)
  const int qrow = r0 + (lane & 15);
  const uint32_t q_lane = qa + qrow * HD * 2;
  const int q_sw = (row0 + qrow) & 7;
  const int q_pc = lane >> 4;
  const int kkey = (lane & 7) + ((lane >> 4) << 3);
  const int k_pc = (lane >> 3) & 1;
  const int vkey = (lane & 7) + (((lane >> 3) & 1) << 3);
  const int v_pc = lane >> 4;

  bool first = true;
#pragma unroll 1
  for (int kb = k0; kb < k1 || first; kb += 64) {
    const int nk = max(0, min(64, k1 - kb));
    if (tid == 0) {
      fence_proxy_async_smem();
      const uint32_t bytes = 2u * (uint32_t)nk * HD * 2u + (first ? (uint32_t)(nrows * HD * 2) : 0u);
      mbar_arrive_expect_tx(att_bar, bytes);
      if (first) bulk_g2s(qa, qg, (uint32_t)nrows * HD * 2, att_bar, pol);
      if (nk > 0) {
        bulk_g2s(ka, kg + (size_t)kb * HD, (uint32_t)nk * HD * 2, att_bar, pol);
        bulk_g2s(va, vg + (size_t)kb * HD, (uint32_t)nk * HD * 2, att_bar, pol);
      }
    }
    {
      const bool w = wait_ab(att_bar, c.att_count & 1, budget, &ctl->abort);
      if (!w) fail(c, E_ATT);
      if (!compute_vote(c, w)) {
        c.ok = false;
        return;
      }
    }
    ++c.att_count;
    {
      // Keys past nk in the last 16-key tile get zero V rows, and query rows
      // past the block get zero q rows, so no stale (possibly non-finite)
      // shared memory meets a zero weight.
      const int nk16 = (nk + 15) & ~15;
      bool synced = false;
      if (nk16 > nk) {
        uint4* zr = reinterpret_cast<uint4*>(vs_ + (size_t)nk * HD * 2);
#pragma unroll 1
        for (int i = tid; i < (nk16 - nk) * HD * 2 / 16; i += kComputeWarps * 32) zr[i] = make_uint4(0u, 0u, 0u, 0u);
        synced = true;
      }
      if (first && nrows < 64) {
        uint4* zq = reinterpret_cast<uint4*>(qs + (size_t)nrows * HD * 2);
#pragma unroll 1
        for (int i = tid; i < (64 - nrows) * HD * 2 / 16; i += kComputeWarps * 32) zq[i] = make_uint4(0u, 0u, 0u, 0u);
        synced = true;
      }
      if (synced) compute_sync();
    }
    first = false;
    const int ksw = kb & 7;   // K/V rows are swizzled by their absolute row (kb is a multiple of 16)
#pragma unroll 1
    for (int kt = 0; kt < nk; kt += 16) {
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      const uint32_t k_lane = ka + (kt + kkey) * HD * 2;
      const int k_sw = (kt + kkey + ksw) & 7;
#pragma unroll 2
      for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
        ldsm_x4(q_lane + (((2 * kk + q_pc) ^ q_sw) << 4), a0, a1, a2, a3);
        ldsm_x4(k_lane + (((2 * kk + k_pc) ^ k_sw) << 4), b0, b1, b2, b3);
        mma16816(s[0], a0, a1, a2, a3, b0, b1);
        mma16816(s[1], a0, a1, a2, a3, b2, b3);
      }
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kt + 8 * t + 2 * (lane & 3) + (e & 1);
          s[t][e] = key < nk ? s[t][e] * sl2 : -INFINITY;
          mx[e >> 1] = fmaxf(mx[e >> 1], s[t][e]);
        }
      }
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 1));
        mx[h2] = fmaxf(mx[h2], __shfl_xor_sync(0xffffffffu, mx[h2], 2));
      }
      float corr[2], mnew[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        mnew[h2] = fmaxf(m_r[h2], mx[h2]);
        corr[h2] = (m_r[h2] == -INFINITY) ? 0.f : exp2f(m_r[h2] - mnew[h2]);
        m_r[h2] = mnew[h2];
        l_r[h2] *= corr[h2];
      }
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float pe = (s[t][e] == -INFINITY) ? 0.f : exp2f(s[t][e] - mnew[e >> 1]);
          s[t][e] = pe;
          l_r[e >> 1] += pe;
        }
#pragma unroll
      for (int i = 0; i < DT; ++i) {
        o[i][0] *= corr[0]; o[i][1] *= corr[0];
        o[i][2] *= corr[1]; o[i][3] *= corr[1];
      }
      const uint32_t pa0 = pack_bf16(s[0][0], s[0][1]);
      const uint32_t pa1 = pack_bf16(s[0][2], s[0][3]);
      const uint32_t pa2 = pack_bf16(s[1][0], s[1][1]);
      const uint32_t pa3 = pack_bf16(s[1][2], s[1][3]);
      const uint32_t v_lane = va + (kt + vkey) * HD * 2;
      const int v_sw = (kt + vkey + ksw) & 7;
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(v_lane + (((2 * dp + v_pc) ^ v_sw) << 4), b0, b1, b2, b3);
        mma16816(o[2 * dp], pa0, pa1, pa2, pa3, b0, b1);
        mma16816(o[2 * dp + 1], pa0, pa1, pa2, pa3, b2, b3);
      }
    }
    fence_proxy_async_smem();
    compute_sync();   // K/V tiles are reused by the next key block
  }
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    l_r[h2] += __shfl_xor_sync(0xffffffffu, l_r[h2], 1);
    l_r[h2] += __shfl_xor_sync(0xffffffffu, l_r[h2], 2);
  }
  tmark(c, 1);
  // Stage (o, m, l) of rows r and r + 8 (row r goes to owner r / 8), then one
  // bulk copy per owner into its receive slot `rank`.
#pragma unroll
  for (int h2 = 0; h2 < 2; ++h2) {
    const int r = r0 + (lane >> 2) + 8 * h2;
    float* dst = stg + r * RWP + 2 * (lane & 3);
#pragma unroll
    for (int i = 0; i < DT; ++i) *reinterpret_cast<float2*>(dst + 8 * i) = make_float2(o[i][2 * h2], o[i][2 * h2 + 1]);
    if ((lane & 3) == 0) *reinterpret_cast<float2*>(stg + r * RWP + HD) = make_float2(m_r[h2], l_r[h2]);
  }
  fence_proxy_async_smem();
  compute_sync();
  if (tid < kClusterSize) {
    // one thread per owner issues that owner's copy
    const uint32_t blk8 = 8u * RWP * 4u;
    const uint32_t recv_local = smem_u32(rb), bar_local = smem_u32(&ctl->recv);
    bulk_s2cluster(map_shared_rank(recv_local + (uint32_t)rank * blk8, tid), smem_u32(stg) + (uint32_t)tid * blk8,
                   blk8, map_shared_rank(bar_local, tid));
  }
  tmark(c, 2);
  {
    const bool w = wait_ab(smem_u32(&ctl->recv), c.recv_count & 1, budget, &ctl->abort);
    if (!w) fail(c, E_RECV);
    if (!compute_vote(c, w)) {
      c.ok = false;
      return;
    }
  }
  ++c.recv_count;
  tmark(c, 3);
  // Combine the 8 key ranges for rows 8*rank .. +7 of the block.
  {
    constexpr int SEGS = HD / 8;
    const int rloc = tid / 16, seg = tid % 16;
    const int rblk = 8 * rank + rloc;
    if (seg < SEGS && rblk < nrows) {
      const float* src = rb + rloc * RWP;
      // every sender's (m, l) first (eight loads in flight), then its o terms
      float2 ml[kClusterSize];
#pragma unroll
      for (int s = 0; s < kClusterSize; ++s) ml[s] = *reinterpret_cast<const float2*>(src + s * 8 * RWP + HD);
      float M = -INFINITY;
#pragma unroll
      for (int s = 0; s < kClusterSize; ++s) M = fmaxf(M, ml[s].x);
      float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < kClusterSize; ++s) {
        const float* sr = src + s * 8 * RWP;
        const float ls = ml[s].y;
        const float wgt = ls == 0.f ? 0.f : exp2f(ml[s].x - M);
        L = fmaf(ls, wgt, L);
        const float4 x0 = *reinterpret_cast<const float4*>(sr + 8 * seg);
        const float4 x1 = *reinterpret_cast<const float4*>(sr + 8 * seg + 4);
        acc[0] = fmaf(x0.x, wgt, acc[0]); acc[1] = fmaf(x0.y, wgt, acc[1]);
        acc[2] = fmaf(x0.z, wgt, acc[2]); acc[3] = fmaf(x0.w, wgt, acc[3]);
        acc[4] = fmaf(x1.x, wgt, acc[4]); acc[5] = fmaf(x1.y, wgt, acc[5]);
        acc[6] = fmaf(x1.z, wgt, acc[6]); acc[7] = fmaf(x1.w, wgt, acc[7]);
      }
      const float inv = 1.0f / L;
      const int R = row0 + rblk;
      const int head = grp * G + R / T, t = R % T;
      uint32_t pk[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) pk[i] = pack_bf16(acc[2 * i] * inv, acc[2 * i + 1] * inv);
      *reinterpret_cast<uint4*>(p.o_act + (size_t)(l & 1) * kRows * p.Hq * HD + act64_off(t, head * HD + 8 * seg)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

__device__ __forceinline__ void phase_attn(Ctx& c, int l) {
  const StepParams& p = *c.p;
  if (!c.ok) return;
  const int units = p.Hkv * p.att_blocks;
  if (c.cluster >= units) return;
  wait_flag(c, F_QKV);
  bool more = false;
  for (int u = c.cluster; u < units; u += p.n_clusters) {
    if (more) {
      // A second unit on this cluster reuses shared memory: every CTA of the
      // cluster must be done with the first one before anyone sends again.
      fence_proxy_async_smem();
      compute_sync();
      if (c.tid == 0) {
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        for (int r = 0; r < kClusterSize; ++r) mbar_arrive_cluster(smem_u32(&c.ctl->xsync), r);
      }
      {
        const bool w = wait_ab(smem_u32(&c.ctl->xsync), c.xs_count & 1, p.spin_budget, &c.ctl->abort);
        if (!w) fail(c, E_RECV);
        if (!compute_vote(c, w)) {
          c.ok = false;
          return;
        }
      }
      ++c.xs_count;
    }
    if (p.hd == 128) attention_unit<128>(c, l, u / p.att_blocks, u % p.att_blocks);
    else attention_unit<64>(c, l, u / p.att_blocks, u % p.att_blocks);
    if (!c.ok) return;
    more = true;
  }
}

// o_proj / down: gated residual on the owned columns, two threads per row t
// (each half of the owned column pairs); z for the next linear, row sum of
// squares.  Operands of the epilogue are fetched before the MMAs finish.
__device__ __forceinline__ void residual_phase(Ctx& c, int g, int f_in, int l, const uint16_t* act,
                                            const float* h_old, float* h_new, const float* gate,
                                            const float* sc, const float* shift, uint16_t* z, float* sumsq) {
  // h_old == nullptr: the residual rows are this thread's registers (the
  // previous residual phase ran on the same owners and thread mapping);
  // h_new == nullptr: the new rows stay in registers only
  if (!c.ok) return;
  const GemmView v = gemm_view(c, g);
  if (v.ng == 0) return;
  arm_recv(c, v);
  const int T = c.p->T, d = c.p->d;
  const int tid = c.tid;
  const int t = tid >> 1, hf = tid & 1;
  const int npair = v.own / 2;
  const int p0 = hf ? npair / 2 : 0, p1 = hf ? npair : npair / 2;
  const int hc0 = v.base + 2 * p0;
  const int np = min(p1 - p0, (d - hc0) / 2);
  float2 ho[kMaxPairs], gt[kMaxPairs], sv[kMaxPairs];
#pragma unroll
  for (int k = 0; k < kMaxPairs; ++k) {
    const int hc = hc0 + 2 * k;
    ho[k] = gt[k] = sv[k] = make_float2(0.f, 0.f);
    if (k < np) {
      gt[k] = *reinterpret_cast<const float2*>(gate + hc);
      // gate x row scale of the linear (exactly the gate for bf16 weights)
      const float2 ws = wscale2(c, g, l, v.pbase + 2 * (p0 + k));
      gt[k].x *= ws.x;
      gt[k].y *= ws.y;
      if (z != nullptr) sv[k] = *reinterpret_cast<const float2*>((t == kBiasRow ? shift : sc) + hc);
    }
  }
  wait_flag(c, f_in, act + (size_t)(v.ks * v.nchunk) * (kRows * 64), v.nchunk);
  tmark(c, 11);
  // global residual rows (first layer of a launch) were stored before an
  // earlier hand-off: visible after the wait
#pragma unroll
  for (int k = 0; k < kMaxPairs; ++k)
    if (k < np && t < T)
      ho[k] = h_old != nullptr ? *reinterpret_cast<const float2*>(h_old + (size_t)t * d + hc0 + 2 * k) : c.hres[k];
  push_send(c, v);
  push_wait(c);
  if (!c.ok) return;
  const float* rb = reinterpret_cast<const float*>(c.work + v.recv_off);
  tmark(c, 8);
  float2 acc[kMaxPairs];
#pragma unroll
  for (int k = 0; k < kMaxPairs; ++k)
    acc[k] = (k < np && t < T) ? (v.KS == kClusterSize ? recv_sum2n<kClusterSize>(rb, v.ownp, t, 2 * (p0 + k))
                                                        : recv_sum2(rb, v.KS, v.ownp, t, 2 * (p0 + k)))
                               : make_float2(0.f, 0.f);
  tmark(c, 9);
  float sq = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxPairs; ++k) {
    if (k >= np) break;
    const int hc = hc0 + 2 * k;
    if (t < T) {
      const float2 a = acc[k];
      const float n0 = fmaf(gt[k].x, a.x, ho[k].x), n1 = fmaf(gt[k].y, a.y, ho[k].y);
      c.hres[k] = make_float2(n0, n1);
      if (h_new != nullptr) *reinterpret_cast<float2*>(h_new + (size_t)t * d + hc) = make_float2(n0, n1);
      sq = fmaf(n0, n0, fmaf(n1, n1, sq));
      if (z != nullptr)
        *reinterpret_cast<uint32_t*>(z + act64_off(t, hc)) = pack_bf16(n0 * (1.0f + sv[k].x), n1 * (1.0f + sv[k].y));
    } else if (t == kBiasRow && z != nullptr) {
      *reinterpret_cast<uint32_t*>(z + act64_off(kBiasRow, hc)) = pack_bf16(sv[k].x, sv[k].y);
    }
  }
  sq += __shfl_xor_sync(0xffffffffu, sq, 1);
  if (hf == 0 && t < T) sumsq[c.cta * kRows + t] = sq;
  tmark(c, 10);
}

// gate_up: reduce, rstd + shift row, SwiGLU -> u (bf16, ACT64).  The owned
// columns hold own/2 gate rows then own/2 matching up rows.
__device__ __forceinline__ void phase_gu(Ctx& c, int step, int l) {
  if (!c.ok) return;
  const StepParams& p = *c.p;
  const GemmView v = gemm_view(c, G_GU);
  if (v.ng == 0) return;
  arm_recv(c, v);
  wait_flag(c, F_ZF, p.z_f + (size_t)(l & 1) * kRows * p.d + (size_t)(v.ks * v.nchunk) * (kRows * 64), v.nchunk);
  tmark(c, 11);
  load_rstd(c, p.sumsq_f);
  push_send(c, v);
  push_wait(c);
  if (!c.ok) return;
  const int T = p.T, F = p.F;
  const int uown = v.own / 2;
  const PairRows pa = pair_rows(c.tid, uown / 2);
  const int uc = v.base + 2 * pa.pr;
  if (!pa.active || uc >= F) return;
  const float* rb = reinterpret_cast<const float*>(c.work + v.recv_off);
  const float* rstd = c.ctl->rstd;
  uint16_t* u_act = p.u_act + (size_t)(l & 1) * kRows * F;
  const int lg = 2 * pa.pr, lu = uown + 2 * pa.pr;
  const float2 sg = wscale2(c, G_GU, l, v.pbase + lg), su = wscale2(c, G_GU, l, v.pbase + lu);
  tmark(c, 8);
  // instruction-bound row loop: the plan's split (two ways) gets a copy
  // without predicated receive slots
  auto rows = [&](auto ksn) {
    constexpr int N = decltype(ksn)::value;
    const float2 bg = N > 0 ? recv_sum2n<(N > 0 ? N : 1)>(rb, v.ownp, kBiasRow, lg)
                            : recv_sum2(rb, v.KS, v.ownp, kBiasRow, lg);
    const float2 bu = N > 0 ? recv_sum2n<(N > 0 ? N : 1)>(rb, v.ownp, kBiasRow, lu)
                            : recv_sum2(rb, v.KS, v.ownp, kBiasRow, lu);
#pragma unroll 1
    for (int t = pa.t0; t < T; t += pa.dt) {
      const float2 ag = N > 0 ? recv_sum2n<(N > 0 ? N : 1)>(rb, v.ownp, t, lg) : recv_sum2(rb, v.KS, v.ownp, t, lg);
      const float2 au = N > 0 ? recv_sum2n<(N > 0 ? N : 1)>(rb, v.ownp, t, lu) : recv_sum2(rb, v.KS, v.ownp, t, lu);
      const float rs = rstd[t];
      const float g0 = fmaf(rs, ag.x, bg.x) * sg.x, g1 = fmaf(rs, ag.y, bg.y) * sg.y;
      const float u0 = fmaf(rs, au.x, bu.x) * su.x, u1 = fmaf(rs, au.y, bu.y) * su.y;
      const float v0 = __fdividef(g0, 1.0f + __expf(-g0)) * u0;
      const float v1 = __fdividef(g1, 1.0f + __expf(-g1)) * u1;
      *reinterpret_cast<uint32_t*>(u_act + act64_off(t, uc)) = pack_bf16(v0, v1);
    }
  };
  if (v.KS == 2) rows(std::integral_constant<int, 2>{});
  else rows(std::integral_constant<int, 0>{});
}

// In-proj: h = x W_in^T for the residual columns this CTA owns in the down
// projection (same owners as sumsq_a); z_a for layer0.
__device__ __forceinline__ void phase_inproj(Ctx& c, int step) {
  if (!c.ok) return;
  const StepParams& p = *c.p;
  const GemmView v = gemm_view(c, G_DOWN);
  if (v.ng == 0) return;
  wait_flag(c, F_X);   // the previous step's Euler update of the whole chunk
  const int T = p.T, A = p.A, d = p.d, own = v.own, base = v.base;
  const int tid = c.tid;
  float* xs = reinterpret_cast<float*>(c.work);            // [T][A]
  float* ws = xs + T * A;                                   // [own][A]
  float* sq = ws + own * A;                                 // [T][own/2]
  {
    const float2* x2 = reinterpret_cast<const float2*>(p.x);
    const int n2 = T * A / 2;
    // unrolled: several batches of loads in flight (same stores)
#pragma unroll 4
    for (int i = tid; i < n2; i += 4 * 128) {
      float2 xv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) xv[j] = i + 128 * j < n2 ? x2[i + 128 * j] : make_float2(0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (i + 128 * j < n2) *reinterpret_cast<float2*>(xs + 2 * (i + 128 * j)) = xv[j];
    }
    const uint16_t* w = p.w_in + (size_t)base * A;
    const int nw = min(own, d - base) * A;
#pragma unroll 4
    for (int i = tid; i < own * A; i += 4 * 128) {
      uint16_t wv[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) wv[j] = i + 128 * j < nw ? w[i + 128 * j] : (uint16_t)0;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (i + 128 * j < own * A) ws[i + 128 * j] = __uint_as_float((uint32_t)wv[j] << 16);
    }
  }
  tmark(c, 8);
  compute_sync();
  tmark(c, 9);
  const float* s_a = mod_vec(p, step, p.layer0, 0);
  const float* b_a = mod_vec(p, step, p.layer0, 1);
  const int npair = own / 2;
  const PairRows pa = pair_rows(tid, npair);
  const int hc = base + 2 * pa.pr;
  if (pa.active && hc < d) {
    float* h_a = p.h_a;
    uint16_t* z_a = p.z_a + (size_t)(p.layer0 & 1) * kRows * d;
    const float2 sa = *reinterpret_cast<const float2*>(s_a + hc);
    const float* w0 = ws + (2 * pa.pr) * A;
    const float* w1 = w0 + A;
    if (pa.t0 == 0)
      *reinterpret_cast<uint32_t*>(z_a + act64_off(kBiasRow, hc)) = pack_bf16(b_a[hc], b_a[hc + 1]);
#pragma unroll 1
    for (int t = pa.t0; t < T; t += pa.dt) {
      const float* xr = xs + t * A;
      float a0 = 0.f, a1 = 0.f, c0 = 0.f, c1 = 0.f;
      int k = 0;
      // unrolled for independent loads; each accumulator's order is unchanged
#pragma unroll 4
      for (; k + 2 <= A; k += 2) {
        a0 = fmaf(xr[k], w0[k], a0);
        a1 = fmaf(xr[k], w1[k], a1);
        c0 = fmaf(xr[k + 1], w0[k + 1], c0);
        c1 = fmaf(xr[k + 1], w1[k + 1], c1);
      }
      if (k < A) {
        a0 = fmaf(xr[k], w0[k], a0);
        a1 = fmaf(xr[k], w1[k], a1);
      }
      a0 += c0;
      a1 += c1;
      *reinterpret_cast<float2*>(h_a + (size_t)t * d + hc) = make_float2(a0, a1);
      *reinterpret_cast<uint32_t*>(z_a + act64_off(t, hc)) = pack_bf16(a0 * (1.0f + sa.x), a1 * (1.0f + sa.y));
      sq[t * npair + pa.pr] = fmaf(a0, a0, a1 * a1);
    }
  } else if (pa.active) {
#pragma unroll 1
    for (int t = pa.t0; t < T; t += pa.dt) sq[t * npair + pa.pr] = 0.f;
  }
  tmark(c, 10);
  compute_sync();
  if (tid < T) {
    float s = 0.f;
#pragma unroll 1
    for (int pr = 0; pr < npair; ++pr) s += sq[tid * npair + pr];
    p.sumsq_a[c.cta * kRows + tid] = s;
  }
}

// Final AdaRMSNorm (s_o, b_o) + out-proj + Euler: items (t, a) in order, a
// contiguous range per warp; the warp keeps y(t) in registers and evaluates
// up to 4 actions at a time.
__device__ __forceinline__ void phase_outproj(Ctx& c, int step) {
  if (!c.ok) return;
  wait_flag(c, F_Z);   // every residual column and its row sums
  const StepParams& p = *c.p;
  const int T = p.T, A = p.A, d = p.d, n_ctas = p.n_ctas;
  const int lane = c.lane;
  const float eps = p.eps, dt = p.dt;
  const float* s_o = p.mod + (size_t)step * p.n_mod + (size_t)6 * p.L * d;
  const float* b_o = s_o + d;
  const float* h_a = p.h_a;
  const float* sumsq = p.sumsq_a;
  const uint16_t* w_out = p.w_out;
  const float* out_bias = p.out_bias;
  float* vbuf = p.vbuf;
  float* x = p.x;
  const bool update = p.update_x != 0;
  const int nw = n_ctas * kComputeWarps;
  const int gw = c.cta * kComputeWarps + (c.warp - 2);
  const int total = T * A;
  const int per = (total + nw - 1) / nw;
  const int i0 = gw * per, i1 = min(total, i0 + per);
  // Lane l takes inputs 256 c + 8 l .. + 7 (c < 4, d <= 1024): one 16-byte
  // load per 8 weights, and every load of a row or a weight pair is in flight
  // at once (the per-element loop had one L2 round trip per few loads).
  constexpr int kC = 4;
  float y[8 * kC];
  int it = i0;
#pragma unroll 1
  while (it < i1) {
    const int t = it / A;
    const int iend = min(i1, (t + 1) * A);
    {
      float q6[kMaxClusters * kClusterSize / 32];
#pragma unroll
      for (int j = 0; j < kMaxClusters * kClusterSize / 32; ++j) {
        const int q = lane + 32 * j;
        q6[j] = q < n_ctas ? sumsq[q * kRows + t] : 0.f;
      }
      float s = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxClusters * kClusterSize / 32; ++j) s += q6[j];
      for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const float rs = 1.0f / sqrtf(s / (float)d + eps);
      // one chunk per wave (its six loads in flight together)
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const int k0 = 256 * c + 8 * lane;
        float4 hv[2], sv[2], bv[2];
        if (k0 < d) {
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            hv[j] = *reinterpret_cast<const float4*>(h_a + (size_t)t * d + k0 + 4 * j);
            sv[j] = *reinterpret_cast<const float4*>(s_o + k0 + 4 * j);
            bv[j] = *reinterpret_cast<const float4*>(b_o + k0 + 4 * j);
          }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float4 h4 = hv[j], s4 = sv[j], b4 = bv[j];
          float* yy = y + 8 * c + 4 * j;
          const bool in = k0 < d;
          yy[0] = in ? fmaf(h4.x * rs, 1.0f + s4.x, b4.x) : 0.f;
          yy[1] = in ? fmaf(h4.y * rs, 1.0f + s4.y, b4.y) : 0.f;
          yy[2] = in ? fmaf(h4.z * rs, 1.0f + s4.z, b4.z) : 0.f;
          yy[3] = in ? fmaf(h4.w * rs, 1.0f + s4.w, b4.w) : 0.f;
        }
      }
    }
    if (it == i0) tmark(c, 8);
#pragma unroll 1
    for (; it < iend; it += 2) {
      const bool two = it + 1 < iend;
      const uint16_t* w = w_out + (size_t)(it - t * A) * d;
      uint4 w0[kC], w1[kC];
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const int k0 = 256 * c + 8 * lane;
        w0[c] = k0 < d ? *reinterpret_cast<const uint4*>(w + k0) : make_uint4(0u, 0u, 0u, 0u);
        w1[c] = (two && k0 < d) ? *reinterpret_cast<const uint4*>(w + d + k0) : make_uint4(0u, 0u, 0u, 0u);
      }
      float dot0 = 0.f, dot1 = 0.f;
#pragma unroll
      for (int c = 0; c < kC; ++c) {
        const uint32_t a[4] = {w0[c].x, w0[c].y, w0[c].z, w0[c].w};
        const uint32_t b[4] = {w1[c].x, w1[c].y, w1[c].z, w1[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dot0 = fmaf(y[8 * c + 2 * e], __uint_as_float(a[e] << 16), dot0);
          dot0 = fmaf(y[8 * c + 2 * e + 1], __uint_as_float(a[e] & 0xFFFF0000u), dot0);
          dot1 = fmaf(y[8 * c + 2 * e], __uint_as_float(b[e] << 16), dot1);
          dot1 = fmaf(y[8 * c + 2 * e + 1], __uint_as_float(b[e] & 0xFFFF0000u), dot1);
        }
      }
      for (int o = 16; o; o >>= 1) {
        dot0 += __shfl_xor_sync(0xffffffffu, dot0, o);
        dot1 += __shfl_xor_sync(0xffffffffu, dot1, o);
      }
      if (lane < 2 && it + lane < iend) {
        const int a = it + lane - t * A;
        const float vv = (lane == 0 ? dot0 : dot1) + (out_bias ? out_bias[a] : 0.f);
        vbuf[(size_t)t * A + a] = vv;
        if (update) x[(size_t)t * A + a] = fmaf(dt, vv, x[(size_t)t * A + a]);
      }
    }
    it = iend;   // the 2-wide steps may overshoot the token boundary
    tmark(c, 9);
  }
}

__device__ __forceinline__ void compute_main(Ctx& c) {
  const StepParams& p = *c.p;
  const int L = p.L, d = p.d;
  const size_t zs = (size_t)kRows * d;
  const bool busy_qkv = gemm_view(c, G_QKV).ng > 0, busy_o = gemm_view(c, G_O).ng > 0,
             busy_gu = gemm_view(c, G_GU).ng > 0, busy_down = gemm_view(c, G_DOWN).ng > 0;
  const bool busy_att = c.cluster < p.Hkv * p.att_blocks;
  for (int s = p.step0; s < p.step1 && c.ok; ++s) {
    if (p.do_inproj) {
      phase_inproj(c, s);
      signal(c, F_Z, busy_down);
    }
    for (int l = p.layer0; l < p.layer1 && c.ok; ++l) {
      const size_t par = (size_t)(l & 1);
      phase_qkv(c, s, l);
      signal(c, F_QKV, busy_qkv);
      phase_attn(c, l);
      signal(c, F_O, busy_att);
      // h lives in the owners' registers between the two residual phases
      // and across layers; it is read from memory at the first layer of a
      // launch and stored after the last (the out-projection and the next
      // launch read it there)
      residual_phase(c, G_O, F_O, l, p.o_act + par * kRows * p.Hq * p.hd,
                     (l == p.layer0 || !p.h_regs) ? p.h_a : nullptr,
                     (p.store_mid || !p.h_regs) ? p.h_b : nullptr, mod_vec(p, s, l, 2),
                     mod_vec(p, s, l, 3), mod_vec(p, s, l, 4), p.z_f + par * zs, p.sumsq_f);
      signal(c, F_ZF, busy_o);
      phase_gu(c, s, l);
      signal(c, F_U, busy_gu);
      {
        const bool next = l + 1 < L;
        residual_phase(c, G_DOWN, F_U, l, p.u_act + par * kRows * p.F, p.h_regs ? nullptr : p.h_b,
                       (l + 1 == p.layer1 || !p.h_regs) ? p.h_a : nullptr,
                       mod_vec(p, s, l, 5),
                       next ? mod_vec(p, s, l + 1, 0) : nullptr, next ? mod_vec(p, s, l + 1, 1) : nullptr,
                       next ? p.z_a + (1 - par) * zs : nullptr, p.sumsq_a);
      }
      signal(c, F_Z, busy_down);
    }
    if (p.do_outproj) {
      phase_outproj(c, s);
      signal(c, F_X, true);
    }
  }
}

}  // namespace

// kWide: quantised weights (two widening warps); otherwise bf16 weights only.
template <bool kWide>
__global__ void __launch_bounds__(kWide ? kStepThreads : kThreads, 1)
    step_kernel(const __grid_constant__ StepParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem;
  uint8_t* work = smem + kRingBytes;
  Ctrl* ctl = reinterpret_cast<Ctrl*>(work + kWorkBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int cluster = cta / kClusterSize;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRingSlots; ++s) {
      mbar_init(smem_u32(&ctl->full[s]), 1);
      mbar_init(smem_u32(&ctl->empty[s]), 1);
      mbar_init(smem_u32(&ctl->conv[s]), 32 * kConvWarps);
    }
    mbar_init(smem_u32(&ctl->act_full), 1);
    mbar_init(smem_u32(&ctl->mma_done), 1);
    mbar_init(smem_u32(&ctl->recv), 1);
    mbar_init(smem_u32(&ctl->att), 1);
    mbar_init(smem_u32(&ctl->drain), 1);
    mbar_init(smem_u32(&ctl->xsync), kClusterSize);
    ctl->abort = 0;
    for (int g = 0; g < 4; ++g) ctl->views[g] = compute_view(p, g, cluster, (int)cluster_rank());
    // writer CTAs of each hand-off: the busy clusters of the phase
    const int units = p.Hkv * p.att_blocks;
    ctl->writers[F_Z] = (uint32_t)(kClusterSize * p.g[G_DOWN].busy_clusters);
    ctl->writers[F_ZF] = (uint32_t)(kClusterSize * p.g[G_O].busy_clusters);
    ctl->writers[F_QKV] = (uint32_t)(kClusterSize * p.g[G_QKV].busy_clusters + (p.stall_test ? 1 : 0));
    ctl->writers[F_U] = (uint32_t)(kClusterSize * p.g[G_GU].busy_clusters);
    ctl->writers[F_O] = (uint32_t)(kClusterSize * min(units, p.n_clusters));
    ctl->writers[F_X] = (uint32_t)p.n_ctas;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // Every CTA of the cluster must have initialised its barriers before any
  // remote store lands on them.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer(p, ring, ctl, cta, cluster);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(p, ring, work, ctl, tmem, cluster);
    __syncwarp();
  } else if (warp >= 2 + kComputeWarps) {
    if constexpr (kWide) converter(p, ring, ctl, cluster, threadIdx.x - 32 * (2 + kComputeWarps));
  } else {
    Ctx c;
    c.p = &p;
    c.work = work;
    c.ctl = ctl;
    c.tmem = tmem;
    c.cta = cta;
    c.cluster = cluster;
    c.rank = (int)cluster_rank();
    c.tid = threadIdx.x - 64;
    c.warp = warp;
    c.lane = lane;
    c.gemm_count = c.recv_count = c.att_count = c.xs_count = 0;
    c.phase = 0;
    for (int f = 0; f < kNumFlags; ++f) c.ep[f] = 0;
    c.P = p.P_dev[p.b];
    c.ok = true;
    compute_main(c);
    if (!c.ok) ctl->abort = 1;
  }
  tc_fence_before();
  __syncthreads();
  // No CTA may leave while a peer can still store into its shared memory.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

namespace {

bool wide_weights(const StepParams& p) { return (p.wfmt[0] | p.wfmt[1] | p.wfmt[2] | p.wfmt[3]) != 0; }

cudaLaunchConfig_t step_config(int n_ctas, bool wide, cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t cfg = {};
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterSize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(n_ctas, 1, 1);
  cfg.blockDim = dim3(wide ? kStepThreads : kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

}  // namespace

size_t step_smem_bytes() { return kSmemBytes; }

cudaError_t step_max_clusters(int* n_clusters) {
  cudaError_t e = cudaFuncSetAttribute(step_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(step_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  const cudaLaunchConfig_t cfg = step_config(kClusterSize * 32, true, attr);
  return cudaOccupancyMaxActiveClusters(n_clusters, step_kernel<true>, &cfg);
}

cudaError_t launch_step(const StepParams& p, cudaStream_t st) {
  cudaLaunchAttribute attr[1];
  const bool wide = wide_weights(p);
  cudaLaunchConfig_t cfg = step_config(p.n_ctas, wide, attr);
  cfg.stream = st;
  return wide ? cudaLaunchKernelEx(&cfg, step_kernel<true>, p) : cudaLaunchKernelEx(&cfg, step_kernel<false>, p);
}

}  // namespace fm
