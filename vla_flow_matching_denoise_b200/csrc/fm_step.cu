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
//  * The grid is every co-resident cluster of 8 CTAs, one CTA per SM.  The
//    phases of the loop are separated by a grid barrier (release/acquire on a
//    global counter, bounded spin).
//  * Weights dominate the bytes (34.6 MB per layer at d = 1024), so warp 0 of
//    every CTA streams its share of every layer, in consumption order, through
//    a 160 KB shared-memory ring with 1-D bulk (TMA) copies.  The stream runs
//    ahead across phases and barriers; only ring space throttles it.
//  * Each linear is split over clusters by output channels and, inside a
//    cluster, over its 8 CTAs by K (and n-groups).  Warp 1 issues tcgen05.mma
//    with M = 64 token rows (50 valid + the shift row + padding), N = the
//    CTA's channels, accumulating fp32 in TMEM.  The split-K partial sums are
//    reduced in a fixed order through distributed shared memory, so results
//    are bit-reproducible.
//  * AdaRMSNorm is folded into the linears: the owner of a residual column
//    writes z = bf16(h (1 + s)) and, in row 50, the shift b; the consumer
//    linear's epilogue applies rstd(row) to rows 0..49 and adds row 50
//    (= b W^T).  This equals y W^T with y = h rstd (1 + s) + b.
//  * Attention (tiny: 50 queries) uses mma.sync with an online softmax per
//    key split and a log-sum-exp combine across the cluster.
#include <cuda_bf16.h>
#include <cstdint>

#include "fm_internal.h"
#include "fm_launch.h"
#include "fm_ptx.cuh"

namespace fm {

namespace {

constexpr uint32_t kRingBytes = 160 * 1024;

struct Ctrl {
  uint64_t full[kRingSlots];
  uint64_t empty[kRingSlots];
  uint64_t act_full;
  uint64_t mma_done;
  uint64_t xa;        // cluster exchange: partial sums / attention partials
  uint64_t xb;        // cluster exchange: row sums of squares, attention reuse
  uint64_t att;       // attention tile loads
  uint64_t drain;
  uint32_t tmem_slot;
  int abort;
  float rstd[kRows];
  float sq_own[kRows];
};

constexpr size_t kSmemBytes = 1024 + kRingBytes + kWorkBytes + ((sizeof(Ctrl) + 127) / 128) * 128;

// Error codes (bit flags in p.err).
enum : uint32_t {
  E_GRID = 1u << 0,
  E_RING_PROD = 1u << 1,
  E_RING_MMA = 1u << 2,
  E_ACT = 1u << 3,
  E_MMA_DONE = 1u << 4,
  E_XA = 1u << 5,
  E_XB = 1u << 6,
  E_ATT = 1u << 7,
};

__device__ __forceinline__ bool wait_ab(uint32_t bar, uint32_t parity, long long budget,
                                        volatile int* abort) {
  if (mbar_test(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test(bar, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
  return true;
}
__device__ __forceinline__ bool wait_cl(uint32_t bar, uint32_t parity, long long budget,
                                        volatile int* abort) {
  if (mbar_test_cluster(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_test_cluster(bar, parity)) {
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
  return true;
}

// Ring placement shared by producer and consumer: a chunk of `sz` bytes goes
// right after the previous one, or wraps to offset 0 when it does not fit.
__device__ __forceinline__ uint32_t ring_place(uint32_t& pos, uint32_t sz) {
  const uint32_t p = (pos + sz > kRingBytes) ? 0u : pos;
  pos = p + sz;
  return p;
}

__device__ __forceinline__ bool gemm_busy(const GemmPlan& g, int cluster) {
  return cluster < g.busy_clusters;
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&b);
}

// 16-byte piece address inside an ACT64 matrix (row r, columns c .. c+7).
__device__ __forceinline__ uint16_t* act64_piece(uint16_t* base, int r, int c) {
  return base + (size_t)(c >> 6) * (kRows * 64) + (size_t)r * 64 + ((((c & 63) >> 3) ^ (r & 7)) << 3);
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&v)[8]) {
  uint4 u;
  u.x = pack_bf16(v[0], v[1]);
  u.y = pack_bf16(v[2], v[3]);
  u.z = pack_bf16(v[4], v[5]);
  u.w = pack_bf16(v[6], v[7]);
  return u;
}

// Element index inside a row of hd bf16 values stored with 16-byte pieces
// swizzled by (row & 7).
__device__ __forceinline__ int swz(int row, int e) {
  return ((((e >> 3) ^ (row & 7))) << 3) | (e & 7);
}

struct Ctx {
  const StepParams* p;
  uint8_t* ring;
  uint8_t* work;
  Ctrl* ctl;
  uint32_t tmem;
  int cta, cluster, rank;
  int tid;              // 0..127 within the compute warps
  int warp;             // 2..5
  int lane;
  uint32_t gemm_count;  // GEMM phases run (parity of act_full / mma_done)
  uint32_t xa_count, xb_count, att_count;
  uint32_t epoch;       // grid barriers passed
  int P;                // prefix length (read from the device)
  bool ok;
};

__device__ __forceinline__ void compute_sync() { named_bar_sync(1, kComputeWarps * 32); }

__device__ void fail(Ctx& c, uint32_t code) {
  atomicOr(c.p->err, code);
  c.ctl->abort = 1;
  c.ok = false;
}

// Grid barrier among the compute warps of every CTA.
__device__ void grid_sync(Ctx& c) {
  if (!c.ok) return;
  fence_proxy_async_global();
  __threadfence();
  compute_sync();
  if (c.tid == 0) {
    red_release_add(c.p->bar_count, 1u);
    const uint32_t target = (c.epoch + 1) * (uint32_t)c.p->n_ctas;
    const long long t0 = clock64();
    bool good = true;
    while (ld_acquire_u32(c.p->bar_count) < target) {
      if (*(volatile uint32_t*)c.p->err != 0u || clock64() - t0 > c.p->spin_budget) {
        good = false;
        break;
      }
    }
    if (!good) fail(c, E_GRID);
    __threadfence();
    fence_proxy_async_global();
  }
  compute_sync();
  if (*(volatile int*)&c.ctl->abort) c.ok = false;
  ++c.epoch;
}

// Cluster exchange among the compute warps: after it, every CTA of the
// cluster may read what the others wrote to their shared memory before it.
__device__ void cluster_exchange(Ctx& c, uint64_t* bar, uint32_t& count, uint32_t code) {
  if (!c.ok) return;
  compute_sync();
  if (c.tid == 0) {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
    for (int r = 0; r < kClusterSize; ++r) mbar_arrive_cluster(smem_u32(bar), r);
  }
  if (!wait_cl(smem_u32(bar), count & 1, c.p->spin_budget, &c.ctl->abort)) fail(c, code);
  ++count;
}

// ------------------------------------------------------------ producer warp
__device__ void producer(const StepParams& p, uint8_t* ring, Ctrl* ctl, int cta, int cluster) {
  const uint64_t pol = policy_evict_first();
  uint32_t nch[4], bytes[4];
  for (int g = 0; g < 4; ++g) {
    nch[g] = gemm_busy(p.g[g], cluster) ? (uint32_t)p.g[g].nchunk : 0u;
    bytes[g] = p.g[g].chunk_bytes;
  }
  uint32_t st[kRingSlots], en[kRingSlots];
  uint32_t head = 0, tail = 0, pos = 0;
  const uint32_t span0 = p.span_off[cta];
  bool good = true;
  for (int s = p.step0; s < p.step1 && good; ++s) {
    for (int l = p.layer0; l < p.layer1 && good; ++l) {
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
          mbar_arrive_expect_tx(smem_u32(&ctl->full[slot]), sz);
          bulk_g2s(smem_u32(ring + at), src, sz, smem_u32(&ctl->full[slot]), pol);
          src += sz;
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

// ------------------------------------------------------------ MMA warp
__device__ void mma_issuer(const StepParams& p, uint8_t* ring, uint8_t* work, Ctrl* ctl,
                           uint32_t tmem, int cluster) {
  uint32_t nch[4], bytes[4], idesc[4];
  for (int g = 0; g < 4; ++g) {
    nch[g] = gemm_busy(p.g[g], cluster) ? (uint32_t)p.g[g].nchunk : 0u;
    bytes[g] = p.g[g].chunk_bytes;
    idesc[g] = idesc_bf16(kRows, p.g[g].Ng);
  }
  uint32_t it = 0, pos = 0, gemm_count = 0;
  bool good = true;
  const uint32_t a_base = smem_u32(work);
  const uint32_t r_base = smem_u32(ring);
  for (int s = p.step0; s < p.step1 && good; ++s) {
    for (int l = p.layer0; l < p.layer1 && good; ++l) {
      for (int g = 0; g < 4 && good; ++g) {
        if (nch[g] == 0) continue;
        if (!wait_ab(smem_u32(&ctl->act_full), gemm_count & 1, p.spin_budget, &ctl->abort)) {
          good = false;
          break;
        }
        tc_fence_after();
        for (uint32_t c = 0; c < nch[g]; ++c, ++it) {
          const uint32_t at = ring_place(pos, bytes[g]);
          const uint32_t slot = it % kRingSlots;
          if (!wait_ab(smem_u32(&ctl->full[slot]), (it / kRingSlots) & 1, p.spin_budget,
                       &ctl->abort)) {
            good = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            mma_bf16(tmem, desc_sw128(a_base + c * 8192 + k16 * 32),
                     desc_sw128(r_base + at + k16 * 32), idesc[g], (c | k16) != 0);
          mma_commit(smem_u32(&ctl->empty[slot]));
        }
        if (!good) break;
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
  mbar_wait(smem_u32(&ctl->drain), 0, p.spin_budget);
}

// ------------------------------------------------------------ compute warps
// Loads this CTA's K-slice of the activation operand of GEMM g.
__device__ void load_act(Ctx& c, int g, const uint16_t* act) {
  const GemmPlan& gp = c.p->g[g];
  if (c.tid == 0) {
    fence_proxy_async_smem();
    const int ks = c.rank % gp.KS;
    const uint32_t bytes = (uint32_t)gp.nchunk * 8192u;
    const uint64_t pol = policy_evict_last();
    mbar_arrive_expect_tx(smem_u32(&c.ctl->act_full), bytes);
    for (int i = 0; i < gp.nchunk; ++i)
      bulk_g2s(smem_u32(c.work + i * 8192),
               act + (size_t)(ks * gp.nchunk + i) * (kRows * 64), 8192,
               smem_u32(&c.ctl->act_full), pol);
  }
}

// Waits for the MMAs of GEMM g, copies rows 0..50 of the fp32 accumulator
// to the staging area (row stride Ng floats) and opens the cluster exchange.
__device__ void stage_partials(Ctx& c, int g) {
  const GemmPlan& gp = c.p->g[g];
  if (!c.ok) return;
  if (!wait_ab(smem_u32(&c.ctl->mma_done), c.gemm_count & 1, c.p->spin_budget, &c.ctl->abort)) {
    fail(c, E_MMA_DONE);
    return;
  }
  ++c.gemm_count;
  tc_fence_after();
  const int sp = c.warp & 3;
  const int row = 16 * sp + c.lane;
  const bool ok = c.lane < 16 && row <= kBiasRow;
  const uint32_t tb = c.tmem + ((uint32_t)(32 * sp) << 16);
  float* stg = reinterpret_cast<float*>(c.work);
#pragma unroll 1
  for (int cb = 0; cb < gp.Ng; cb += 16) {
    float v[16];
    tmem_ld16(tb + cb, v);
    tmem_ld_wait();
    if (ok) {
      float4* dst = reinterpret_cast<float4*>(stg + (size_t)row * gp.Ng + cb);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  }
  tc_fence_before();
  cluster_exchange(c, &c.ctl->xa, c.xa_count, E_XA);
}

// rstd[t] = (sum of per-cluster partial sums of h^2 / d + eps)^-1/2, rows < T.
__device__ void load_rstd(Ctx& c, const float* sumsq) {
  const StepParams& p = *c.p;
  if (c.tid < p.T) {
    float s = 0.f;
    for (int q = 0; q < p.n_clusters; ++q) s += sumsq[q * kRows + c.tid];
    c.ctl->rstd[c.tid] = 1.0f / sqrtf(s / (float)p.d + p.eps);
  }
  compute_sync();
}

// Writes the cluster's row sums of squares: rank 0 adds the 8 CTAs' partials.
__device__ void publish_sumsq(Ctx& c, float* sumsq) {
  cluster_exchange(c, &c.ctl->xb, c.xb_count, E_XB);
  if (!c.ok) return;
  if (c.rank == 0 && c.tid < c.p->T) {
    const uint32_t a = smem_u32(&c.ctl->sq_own[c.tid]);
    float s = 0.f;
    for (int r = 0; r < kClusterSize; ++r) s += ld_dsmem_f1(map_shared_rank(a, r));
    sumsq[c.cluster * kRows + c.tid] = s;
  }
}

// Residual-column owner: h_new = h_old + gate * acc for 8 columns starting at
// global column hc, row t; writes h_new, z = bf16(h_new (1 + s)) and returns
// sum of squares.
__device__ __forceinline__ float residual8(const float* h_old, float* h_new, uint16_t* z,
                                           const float* gate, const float* sc, int d, int t, int hc,
                                           const float (&acc)[8]) {
  const float4* ho = reinterpret_cast<const float4*>(h_old + (size_t)t * d + hc);
  const float4 h0 = ho[0], h1 = ho[1];
  const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
  float out[8], zv[8], sq = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    out[i] = fmaf(gate[hc + i], acc[i], hv[i]);
    sq = fmaf(out[i], out[i], sq);
  }
  float4* hn = reinterpret_cast<float4*>(h_new + (size_t)t * d + hc);
  hn[0] = make_float4(out[0], out[1], out[2], out[3]);
  hn[1] = make_float4(out[4], out[5], out[6], out[7]);
  if (z != nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) zv[i] = out[i] * (1.0f + sc[hc + i]);
    *reinterpret_cast<uint4*>(act64_piece(z, t, hc)) = pack8_bf16(zv);
  }
  return sq;
}

__device__ __forceinline__ void write_shift_row(uint16_t* z, const float* shift, int hc) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = shift[hc + i];
  *reinterpret_cast<uint4*>(act64_piece(z, kBiasRow, hc)) = pack8_bf16(v);
}

__device__ __forceinline__ const float* mod_vec(const StepParams& p, int step, int l, int which) {
  return p.mod + (size_t)step * p.n_mod + ((size_t)6 * l + which) * p.d;
}

// In-proj: h = x W_in^T for the CTA's residual columns; z_a for layer0.
__device__ void phase_inproj(Ctx& c, int step) {
  const StepParams& p = *c.p;
  // Same column ownership as the down projection: both write sumsq_a.
  const GemmPlan& go = p.g[G_DOWN];
  if (!c.ok) return;
  const bool busy = gemm_busy(go, c.cluster);
  if (busy) {
    const int base = c.cluster * go.NS * go.Ng + (c.rank / go.KS) * go.Ng + (c.rank % go.KS) * go.own;
    const float* s_a = mod_vec(p, step, p.layer0, 0);
    const float* b_a = mod_vec(p, step, p.layer0, 1);
    float sq = 0.f;
    for (int q = 0; q < go.own; q += 8) {
      const int hc = base + q;
      if (hc >= p.d) break;
      if (c.tid < p.T) {
        float acc[8];
        const float* xr = p.x + (size_t)c.tid * p.A;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint16_t* w = p.w_in + (size_t)(hc + i) * p.A;
          float a = 0.f;
          for (int k = 0; k < p.A; ++k) a = fmaf(xr[k], __uint_as_float((uint32_t)w[k] << 16), a);
          acc[i] = a;
        }
        float* hr = p.h_a + (size_t)c.tid * p.d + hc;
        float zv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          hr[i] = acc[i];
          sq = fmaf(acc[i], acc[i], sq);
          zv[i] = acc[i] * (1.0f + s_a[hc + i]);
        }
        *reinterpret_cast<uint4*>(act64_piece(p.z_a, c.tid, hc)) = pack8_bf16(zv);
      } else if (c.tid == kBiasRow) {
        write_shift_row(p.z_a, b_a, hc);
      }
    }
    if (c.tid < p.T) c.ctl->sq_own[c.tid] = sq;
    publish_sumsq(c, p.sumsq_a);
  }
}

// QKV: z_a K-slice x packed W_qkv -> cluster reduce -> rstd, shift row, RoPE
// -> q buffer and the chunk rows of the KV cache.
__device__ void phase_qkv(Ctx& c, int step, int l) {
  const StepParams& p = *c.p;
  const GemmPlan& gp = p.g[G_QKV];
  if (!c.ok || !gemm_busy(gp, c.cluster)) return;
  load_act(c, G_QKV, p.z_a);
  load_rstd(c, p.sumsq_a);
  stage_partials(c, G_QKV);
  if (!c.ok) return;
  const int ng = c.rank / gp.KS, ks = c.rank % gp.KS;
  const int col0 = ks * gp.own;
  const int npair = gp.own / 2;
  const uint32_t stg = smem_u32(c.work);
  const int qn = p.Hq * p.hd, kn = p.Hkv * p.hd;
  const int half = p.hd / 2;
  const int Nc = gp.NS * gp.Ng;
  for (int item = c.tid; item < p.T * npair; item += kComputeWarps * 32) {
    const int t = item / npair, pr = item % npair;
    const int col = col0 + 2 * pr;
    const int n = c.cluster * Nc + ng * gp.Ng + col;
    if (n >= gp.N) continue;
    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
    for (int r = 0; r < gp.KS; ++r) {
      const int peer = ng * gp.KS + r;
      const float2 va = ld_dsmem_f2(map_shared_rank(stg + 4u * (uint32_t)(t * gp.Ng + col), peer));
      const float2 vb = ld_dsmem_f2(map_shared_rank(stg + 4u * (uint32_t)(kBiasRow * gp.Ng + col), peer));
      a0 += va.x; a1 += va.y; b0 += vb.x; b1 += vb.y;
    }
    const float rs = c.ctl->rstd[t];
    const float y0 = fmaf(rs, a0, b0), y1 = fmaf(rs, a1, b1);
    if (n < qn + kn) {
      const bool is_q = n < qn;
      const int nn = is_q ? n : n - qn;
      const int head = nn / p.hd, w = nn % p.hd, i = w >> 1;
      const float cs = p.rope[(t * half + i) * 2], sn = p.rope[(t * half + i) * 2 + 1];
      const float o1 = y0 * cs - y1 * sn;
      const float o2 = y1 * cs + y0 * sn;
      uint16_t* row;
      int rr;
      if (is_q) {
        rr = t;
        row = p.qbuf + ((size_t)head * kRows + t) * p.hd;
      } else {
        rr = c.P + t;
        row = p.kcache + ((((size_t)l * p.B_cap + p.b) * p.Hkv + head) * p.S_max + rr) * p.hd;
      }
      row[swz(rr, i)] = bf16_bits(o1);
      row[swz(rr, i + half)] = bf16_bits(o2);
    } else {
      const int nn = n - qn - kn;
      const int head = nn / p.hd, w = nn % p.hd;
      const int rr = c.P + t;
      uint16_t* row = p.vcache + ((((size_t)l * p.B_cap + p.b) * p.Hkv + head) * p.S_max + rr) * p.hd;
      row[swz(rr, w)] = bf16_bits(y0);
      row[swz(rr, w + 1)] = bf16_bits(y1);
    }
  }
  fence_proxy_async_smem();
}

// GQA attention for the cluster's query head(s); this CTA takes one key range.
template <int HD>
__device__ void attention_head(Ctx& c, int l, int head) {
  const StepParams& p = *c.p;
  constexpr int KSTEPS = HD / 16;
  constexpr int DT = HD / 8;         // n-tiles of the output
  const int G = p.Hq / p.Hkv;
  const int g = head / G;
  const int S = c.P + p.T;
  const int kpc = ((S + kClusterSize * 16 - 1) / (kClusterSize * 16)) * 16;
  const int k0 = c.rank * kpc;
  const int k1 = min(S, k0 + kpc);
  uint8_t* qs = c.work;
  uint8_t* ks_ = c.work + kRows * HD * 2;
  uint8_t* vs_ = ks_ + 64 * HD * 2;
  const uint32_t qa = smem_u32(qs), ka = smem_u32(ks_), va = smem_u32(vs_);
  const uint64_t pol = policy_evict_last();
  const uint16_t* kg = p.kcache + ((((size_t)l * p.B_cap + p.b) * p.Hkv + g) * p.S_max) * HD;
  const uint16_t* vg = p.vcache + ((((size_t)l * p.B_cap + p.b) * p.Hkv + g) * p.S_max) * HD;

  const int w4 = c.warp - 2;               // rows 16*w4 .. +15
  const int r0 = 16 * w4;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);
  float m_r[2] = {-INFINITY, -INFINITY}, l_r[2] = {0.f, 0.f};
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  uint32_t qf[KSTEPS][4];

  bool first = true;
  for (int kb = k0; kb < k1 || first; kb += 64) {
    const int nk = max(0, min(64, k1 - kb));
    if (c.tid == 0) {
      fence_proxy_async_smem();
      uint32_t bytes = 2u * (uint32_t)nk * HD * 2u + (first ? (uint32_t)(kRows * HD * 2) : 0u);
      mbar_arrive_expect_tx(smem_u32(&c.ctl->att), bytes);
      if (first)
        bulk_g2s(qa, p.qbuf + (size_t)head * kRows * HD, kRows * HD * 2, smem_u32(&c.ctl->att), pol);
      if (nk > 0) {
        bulk_g2s(ka, kg + (size_t)kb * HD, (uint32_t)nk * HD * 2, smem_u32(&c.ctl->att), pol);
        bulk_g2s(va, vg + (size_t)kb * HD, (uint32_t)nk * HD * 2, smem_u32(&c.ctl->att), pol);
      }
    }
    if (!wait_ab(smem_u32(&c.ctl->att), c.att_count & 1, p.spin_budget, &c.ctl->abort)) {
      fail(c, E_ATT);
      return;
    }
    ++c.att_count;
    {
      // Keys past nk in the last 16-key tile get zero V rows, so that their
      // zero softmax weights cannot meet stale (possibly non-finite) data.
      const int nk16 = (nk + 15) & ~15;
      if (nk16 > nk) {
        uint4* zr = reinterpret_cast<uint4*>(vs_ + (size_t)nk * HD * 2);
        for (int i = c.tid; i < (nk16 - nk) * HD * 2 / 16; i += kComputeWarps * 32)
          zr[i] = make_uint4(0u, 0u, 0u, 0u);
        compute_sync();
      }
    }
    if (first) {
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int row = r0 + (c.lane & 15);
        const int pc = 2 * kk + (c.lane >> 4);
        ldsm_x4(qa + row * HD * 2 + ((pc ^ (row & 7)) << 4), qf[kk][0], qf[kk][1], qf[kk][2],
                qf[kk][3]);
      }
      first = false;
    }
    for (int kt = 0; kt < nk; kt += 16) {
      float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int key = kt + (c.lane & 7) + ((c.lane >> 4) << 3);
        const int pc = 2 * kk + ((c.lane >> 3) & 1);
        const int gk = kb + key;   // absolute row decides the swizzle
        uint32_t b0, b1, b2, b3;
        ldsm_x4(ka + key * HD * 2 + ((pc ^ (gk & 7)) << 4), b0, b1, b2, b3);
        mma16816(s[0], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
        mma16816(s[1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
      }
      // scale, mask, online softmax (rows lane/4 and lane/4 + 8)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int t = 0; t < 2; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = kt + 8 * t + 2 * (c.lane & 3) + (e & 1);
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
#pragma unroll
      for (int dp = 0; dp < DT / 2; ++dp) {
        const int key = kt + (c.lane & 7) + (((c.lane >> 3) & 1) << 3);
        const int pc = 2 * dp + (c.lane >> 4);
        const int gk = kb + key;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(va + key * HD * 2 + ((pc ^ (gk & 7)) << 4), b0, b1, b2, b3);
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
  // Partials to staging: [64 rows][HD + 4] fp32: o (unnormalised), m, l.
  constexpr int RS = HD + 4;
  float* stg = reinterpret_cast<float*>(c.work);
  compute_sync();   // q tile is dead; staging overlaps it
  {
    const int ra = r0 + (c.lane >> 2), rb = ra + 8;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      const int col = 8 * i + 2 * (c.lane & 3);
      *reinterpret_cast<float2*>(stg + ra * RS + col) = make_float2(o[i][0], o[i][1]);
      *reinterpret_cast<float2*>(stg + rb * RS + col) = make_float2(o[i][2], o[i][3]);
    }
    if ((c.lane & 3) == 0) {
      stg[ra * RS + HD] = m_r[0];
      stg[ra * RS + HD + 1] = l_r[0];
      stg[rb * RS + HD] = m_r[1];
      stg[rb * RS + HD + 1] = l_r[1];
    }
  }
  cluster_exchange(c, &c.ctl->xa, c.xa_count, E_XA);
  if (!c.ok) return;
  // Combine: this CTA finalises rows 8*rank .. +7.
  {
    constexpr int SEGS = HD / 8;
    const int rloc = c.tid / 16, seg = c.tid % 16;
    const int t = 8 * c.rank + rloc;
    if (seg < SEGS && t < p.T) {
      const uint32_t base = smem_u32(stg);
      float mr[kClusterSize], lr[kClusterSize];
      float M = -INFINITY;
#pragma unroll
      for (int r = 0; r < kClusterSize; ++r) {
        const float2 ml = ld_dsmem_f2(map_shared_rank(base + 4u * (uint32_t)(t * RS + HD), r));
        mr[r] = ml.x;
        lr[r] = ml.y;
        M = fmaxf(M, ml.x);
      }
      float L = 0.f, acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int r = 0; r < kClusterSize; ++r) {
        if (lr[r] == 0.f) continue;
        const float wgt = exp2f(mr[r] - M);
        L = fmaf(lr[r], wgt, L);
        const uint32_t a = map_shared_rank(base + 4u * (uint32_t)(t * RS + 8 * seg), r);
        const float4 x0 = ld_dsmem_f4(a), x1 = ld_dsmem_f4(a + 16);
        acc[0] = fmaf(x0.x, wgt, acc[0]); acc[1] = fmaf(x0.y, wgt, acc[1]);
        acc[2] = fmaf(x0.z, wgt, acc[2]); acc[3] = fmaf(x0.w, wgt, acc[3]);
        acc[4] = fmaf(x1.x, wgt, acc[4]); acc[5] = fmaf(x1.y, wgt, acc[5]);
        acc[6] = fmaf(x1.z, wgt, acc[6]); acc[7] = fmaf(x1.w, wgt, acc[7]);
      }
      const float inv = 1.0f / L;
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= inv;
      *reinterpret_cast<uint4*>(act64_piece(p.o_act, t, head * HD + 8 * seg)) = pack8_bf16(acc);
    }
  }
  fence_proxy_async_smem();
}

__device__ void phase_attn(Ctx& c, int l) {
  const StepParams& p = *c.p;
  if (!c.ok) return;
  bool more = false;
  for (int head = c.cluster; head < p.Hq; head += p.n_clusters) {
    if (more) {
      // The staging area is reused: wait until every CTA finished reading it.
      cluster_exchange(c, &c.ctl->xb, c.xb_count, E_XB);
      if (!c.ok) return;
    }
    if (p.hd == 128) attention_head<128>(c, l, head);
    else attention_head<64>(c, l, head);
    if (!c.ok) return;
    more = true;
  }
}

// o_proj / down: reduce the split-K partial sums of the CTA's 8-column
// groups, apply the gated residual, emit z for the next linear and the row
// sums of squares.
__device__ void residual_epilogue(Ctx& c, int g, const float* h_old, float* h_new,
                                  const float* gate, const float* sc, const float* shift,
                                  uint16_t* z, float* sumsq) {
  const StepParams& p = *c.p;
  const GemmPlan& gp = p.g[g];
  const int ng = c.rank / gp.KS, ks = c.rank % gp.KS;
  const uint32_t stg = smem_u32(c.work);
  const int Nc = gp.NS * gp.Ng;
  float sq = 0.f;
  for (int q = 0; q < gp.own; q += 8) {
    const int col = ks * gp.own + q;
    const int hc = c.cluster * Nc + ng * gp.Ng + col;
    if (hc >= p.d) break;
    if (c.tid < p.T) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int r = 0; r < gp.KS; ++r) {
        const uint32_t a = map_shared_rank(stg + 4u * (uint32_t)(c.tid * gp.Ng + col), ng * gp.KS + r);
        const float4 x0 = ld_dsmem_f4(a), x1 = ld_dsmem_f4(a + 16);
        acc[0] += x0.x; acc[1] += x0.y; acc[2] += x0.z; acc[3] += x0.w;
        acc[4] += x1.x; acc[5] += x1.y; acc[6] += x1.z; acc[7] += x1.w;
      }
      sq += residual8(h_old, h_new, z, gate, sc, p.d, c.tid, hc, acc);
    } else if (c.tid == kBiasRow && z != nullptr) {
      write_shift_row(z, shift, hc);
    }
  }
  if (c.tid < p.T) c.ctl->sq_own[c.tid] = sq;
  publish_sumsq(c, sumsq);
}

__device__ void phase_o(Ctx& c, int step, int l) {
  const StepParams& p = *c.p;
  const GemmPlan& gp = p.g[G_O];
  if (!c.ok || !gemm_busy(gp, c.cluster)) return;
  load_act(c, G_O, p.o_act);
  stage_partials(c, G_O);
  if (!c.ok) return;
  residual_epilogue(c, G_O, p.h_a, p.h_b, mod_vec(p, step, l, 2), mod_vec(p, step, l, 3),
                    mod_vec(p, step, l, 4), p.z_f, p.sumsq_f);
  fence_proxy_async_smem();
}

__device__ void phase_down(Ctx& c, int step, int l) {
  const StepParams& p = *c.p;
  const GemmPlan& gp = p.g[G_DOWN];
  if (!c.ok || !gemm_busy(gp, c.cluster)) return;
  load_act(c, G_DOWN, p.u_act);
  stage_partials(c, G_DOWN);
  if (!c.ok) return;
  const bool next = l + 1 < p.L;
  residual_epilogue(c, G_DOWN, p.h_b, p.h_a, mod_vec(p, step, l, 5),
                    next ? mod_vec(p, step, l + 1, 0) : nullptr,
                    next ? mod_vec(p, step, l + 1, 1) : nullptr, next ? p.z_a : nullptr,
                    p.sumsq_a);
  fence_proxy_async_smem();
}

// gate_up: reduce, rstd + shift row, SwiGLU -> u (bf16, ACT64).
__device__ void phase_gu(Ctx& c, int step, int l) {
  const StepParams& p = *c.p;
  const GemmPlan& gp = p.g[G_GU];
  if (!c.ok || !gemm_busy(gp, c.cluster)) return;
  load_act(c, G_GU, p.z_f);
  load_rstd(c, p.sumsq_f);
  stage_partials(c, G_GU);
  if (!c.ok) return;
  const int ng = c.rank / gp.KS, ks = c.rank % gp.KS;
  const int uown = gp.own / 2;                  // u columns owned
  const int npiece = uown / 8;
  const uint32_t stg = smem_u32(c.work);
  const int ubase = (c.cluster * gp.NS + ng) * p.uc + ks * uown;
  const int gcol0 = ks * gp.own;                // gate columns, then up columns
  for (int item = c.tid; item < p.T * npiece; item += kComputeWarps * 32) {
    const int t = item / npiece, q = item % npiece;
    const int uc = ubase + 8 * q;
    if (uc >= p.F) continue;
    float ag[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f}, au[8], bg[8], bu[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) au[i] = bg[i] = bu[i] = 0.f;
    for (int r = 0; r < gp.KS; ++r) {
      const int peer = ng * gp.KS + r;
      const uint32_t rg = map_shared_rank(stg + 4u * (uint32_t)(t * gp.Ng + gcol0 + 8 * q), peer);
      const uint32_t ru = rg + 4u * (uint32_t)uown;
      const uint32_t bgp = map_shared_rank(stg + 4u * (uint32_t)(kBiasRow * gp.Ng + gcol0 + 8 * q), peer);
      const uint32_t bup = bgp + 4u * (uint32_t)uown;
      float4 x;
      x = ld_dsmem_f4(rg); ag[0] += x.x; ag[1] += x.y; ag[2] += x.z; ag[3] += x.w;
      x = ld_dsmem_f4(rg + 16); ag[4] += x.x; ag[5] += x.y; ag[6] += x.z; ag[7] += x.w;
      x = ld_dsmem_f4(ru); au[0] += x.x; au[1] += x.y; au[2] += x.z; au[3] += x.w;
      x = ld_dsmem_f4(ru + 16); au[4] += x.x; au[5] += x.y; au[6] += x.z; au[7] += x.w;
      x = ld_dsmem_f4(bgp); bg[0] += x.x; bg[1] += x.y; bg[2] += x.z; bg[3] += x.w;
      x = ld_dsmem_f4(bgp + 16); bg[4] += x.x; bg[5] += x.y; bg[6] += x.z; bg[7] += x.w;
      x = ld_dsmem_f4(bup); bu[0] += x.x; bu[1] += x.y; bu[2] += x.z; bu[3] += x.w;
      x = ld_dsmem_f4(bup + 16); bu[4] += x.x; bu[5] += x.y; bu[6] += x.z; bu[7] += x.w;
    }
    const float rs = c.ctl->rstd[t];
    float uv[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float gt = fmaf(rs, ag[i], bg[i]);
      const float up = fmaf(rs, au[i], bu[i]);
      uv[i] = gt / (1.0f + expf(-gt)) * up;
    }
    *reinterpret_cast<uint4*>(act64_piece(p.u_act, t, uc)) = pack8_bf16(uv);
  }
  fence_proxy_async_smem();
}

// Final AdaRMSNorm (s_o, b_o) + out-proj + Euler, spread over every warp.
__device__ void phase_outproj(Ctx& c, int step) {
  const StepParams& p = *c.p;
  if (!c.ok) return;
  const float* s_o = p.mod + (size_t)step * p.n_mod + (size_t)6 * p.L * p.d;
  const float* b_o = s_o + p.d;
  const int nw = p.n_ctas * kComputeWarps;
  const int gw = c.cta * kComputeWarps + (c.warp - 2);
  const int total = p.T * p.A;
  const int per = (total + nw - 1) / nw;
  const int i0 = gw * per, i1 = min(total, i0 + per);
  constexpr int MAXV = 32;   // d <= 1024
  float y[MAXV];
  int cur_t = -1;
  for (int it = i0; it < i1; ++it) {
    const int t = it / p.A, a = it % p.A;
    if (t != cur_t) {
      float s = 0.f;
      for (int q = 0; q < p.n_clusters; ++q) s += p.sumsq_a[q * kRows + t];
      const float rs = 1.0f / sqrtf(s / (float)p.d + p.eps);
#pragma unroll
      for (int i = 0; i < MAXV; ++i) {
        const int k = c.lane + 32 * i;
        y[i] = k < p.d ? fmaf(p.h_a[(size_t)t * p.d + k] * rs, 1.0f + s_o[k], b_o[k]) : 0.f;
      }
      cur_t = t;
    }
    float dot = 0.f;
    const uint16_t* w = p.w_out + (size_t)a * p.d;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int k = c.lane + 32 * i;
      if (k < p.d) dot = fmaf(y[i], __uint_as_float((uint32_t)w[k] << 16), dot);
    }
    for (int o = 16; o; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (c.lane == 0) {
      const float v = dot + (p.out_bias ? p.out_bias[a] : 0.f);
      p.vbuf[(size_t)t * p.A + a] = v;
      if (p.update_x) p.x[(size_t)t * p.A + a] = fmaf(p.dt, v, p.x[(size_t)t * p.A + a]);
    }
  }
}

__device__ void compute_main(Ctx& c) {
  const StepParams& p = *c.p;
  for (int s = p.step0; s < p.step1 && c.ok; ++s) {
    if (p.do_inproj) {
      phase_inproj(c, s);
      grid_sync(c);
    }
    for (int l = p.layer0; l < p.layer1 && c.ok; ++l) {
      phase_qkv(c, s, l);
      grid_sync(c);
      phase_attn(c, l);
      grid_sync(c);
      phase_o(c, s, l);
      grid_sync(c);
      phase_gu(c, s, l);
      grid_sync(c);
      phase_down(c, s, l);
      grid_sync(c);
    }
    if (p.do_outproj) {
      phase_outproj(c, s);
      grid_sync(c);
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) step_kernel(const __grid_constant__ StepParams p) {
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
    }
    mbar_init(smem_u32(&ctl->act_full), 1);
    mbar_init(smem_u32(&ctl->mma_done), 1);
    mbar_init(smem_u32(&ctl->xa), kClusterSize);
    mbar_init(smem_u32(&ctl->xb), kClusterSize);
    mbar_init(smem_u32(&ctl->att), 1);
    mbar_init(smem_u32(&ctl->drain), 1);
    ctl->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&ctl->tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  // Every CTA of the cluster must have initialised its barriers before any
  // remote arrive lands on them.
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = ctl->tmem_slot;

  if (warp == 0) {
    if (lane == 0) producer(p, ring, ctl, cta, cluster);
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) mma_issuer(p, ring, work, ctl, tmem, cluster);
    __syncwarp();
  } else {
    Ctx c;
    c.p = &p;
    c.ring = ring;
    c.work = work;
    c.ctl = ctl;
    c.tmem = tmem;
    c.cta = cta;
    c.cluster = cluster;
    c.rank = (int)cluster_rank();
    c.tid = threadIdx.x - 64;
    c.warp = warp;
    c.lane = lane;
    c.gemm_count = c.xa_count = c.xb_count = c.att_count = 0;
    c.epoch = 0;
    c.P = *p.P_dev;
    c.ok = true;
    compute_main(c);
    if (!c.ok) ctl->abort = 1;
  }
  tc_fence_before();
  __syncthreads();
  // No CTA may leave while a peer can still read its shared memory.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

size_t step_smem_bytes() { return kSmemBytes; }

cudaError_t step_max_clusters(int* n_clusters) {
  cudaError_t e = cudaFuncSetAttribute(step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterSize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(kClusterSize * 32, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(n_clusters, step_kernel, &cfg);
}

cudaError_t launch_step(const StepParams& p, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kClusterSize;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(p.n_ctas, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, step_kernel, p);
}

}  // namespace fm
