// Host engine behind include/fm_expert.h: argument checks, the work plan,
// weight packing into the kernel-ready arena, buffers, the prefix cache, the
// per-(batch, steps) CUDA-graph cache and the test hooks.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <map>
#include <string>
#include <utility>
#include <vector>

#include "../../include/fm_expert.h"
#include "fm_batch.h"
#include "fm_internal.h"
#include "fm_launch.h"

using namespace fm;

namespace {

thread_local std::string g_create_error;

}  // namespace

void fm::set_thread_error(const char* msg) { g_create_error = msg; }

namespace {

struct DevBuf {
  void* p = nullptr;
  size_t n = 0;
};

}  // namespace

struct fm_expert {
  fm_config cfg{};
  int device = 0;
  int n_sms = 0;
  int n_clusters = 0;
  int n_ctas = 0;
  int n_mod = 0;
  GemmPlan plan[4]{};
  int att_blocks = 0;
  int q_rows = 0;
  std::string err;
  std::vector<DevBuf> bufs;
  size_t bytes = 0;
  cudaStream_t cap_stream = nullptr;
  // weights
  uint8_t* arena = nullptr;
  uint64_t layer_bytes = 0;
  uint32_t* span_off = nullptr;
  uint8_t* w2_packed = nullptr;
  uint16_t* w1 = nullptr;
  uint16_t* w_in = nullptr;
  uint16_t* w_in_t = nullptr;        // [A][d]: the batched in-proj's transposed copy
  uint16_t* w_out = nullptr;
  float* out_bias = nullptr;
  // E4M3 weights: row scales by packed channel (read by the kernel) and, for
  // fm_get_fp8_weights, the packing tables and the scales in source-row order
  float* wscale = nullptr;           // [L][sc_stride]
  int sc_stride = 0;
  int sc_off[4] = {0, 0, 0, 0};
  std::vector<PackChunk> pack_jobs;
  std::vector<int32_t> pack_rows;
  std::vector<float> row_scale;      // [L][rows of QKV + O + GU + DOWN]
  std::vector<float> nv4_g;          // NVFP4 gate_up: [L][2] tensor scales (gate, up)
  // batched path (the requests of a call advance together, M = B * T rows: B >= 2 on
  // a bf16 handle, every B on a W8A8 handle)
  bool batched = false;
  bool w8a8 = false;                 // E4M3 weights and per-token E4M3 activations (every B batched)
  uint8_t* barena = nullptr;         // per layer: [N/BN][K/64] chunks of each linear (W8A8: [N/BN][K/128])
  uint64_t blayer_bytes = 0;
  uint64_t boff[4] = {0, 0, 0, 0};
  int Mp = 0;                        // padded rows of the batched activations
  uint16_t* bz_a = nullptr;          // ACT128 [Mp/128][d/64]
  uint16_t* bz_f = nullptr;
  uint16_t* bo = nullptr;            // ACT128 [Mp/128][Hq*hd/64]
  uint16_t* bu = nullptr;            // ACT128 [Mp/128][F/64]
  float* bh = nullptr;               // [Mp][d] residual
  uint16_t* bq = nullptr;            // [B_cap][Hkv][q_rows][hd]
  // W8A8: weight scales by GEMM column, activation codes and their row scales
  float* bwscale = nullptr;          // [L][bw_stride]: the four linears' columns in tile order
  int bw_stride = 0;
  int bw_off[4] = {0, 0, 0, 0};
  std::vector<PackChunk> bpack_jobs; // tile chunks and their source rows (fm_get_fp8_weights)
  std::vector<int32_t> bpack_rows;
  uint8_t* bo8 = nullptr;            // ACT8 [Mp/128][Hq*hd/128]
  uint8_t* bu8 = nullptr;            // ACT8 [Mp/128][F/128]
  float* bsa = nullptr;              // [4][Mp]: row scales of z_a, o, z_f, u
  // prefix cache builder (fm_set_prefix_builder / fm_build_prefix)
  int pre_d = 0;                     // backbone hidden width (0: no builder weights)
  uint8_t* pre_arena = nullptr;      // per layer: [Wk; Wv] in [N/BN][d/64] chunks
  uint64_t pre_layer_bytes = 0;
  uint16_t* pre_stage = nullptr;     // ACT128 hidden states of one layer
  uint16_t* pre_rows = nullptr;      // device copy of a host layer input
  float* pre_rope = nullptr;         // [max_prefix][hd/2][2] at positions 0 .. max_prefix-1
  int* pre_zero = nullptr;           // one 0: the position offset of the prefix table
  // buffers
  float* mod = nullptr;
  uint16_t* h1_act = nullptr;
  float* rope = nullptr;
  int* P_dev = nullptr;
  float* x = nullptr;      // [B_cap, T, A]
  float* vbuf = nullptr;   // [B_cap, T, A]
  float* h_a = nullptr;
  float* h_b = nullptr;
  uint16_t* z_a = nullptr;
  uint16_t* z_f = nullptr;
  uint16_t* o_act = nullptr;
  uint16_t* u_act = nullptr;
  float* sumsq_a = nullptr;
  float* sumsq_f = nullptr;
  uint16_t* qbuf = nullptr;
  uint16_t* kcache = nullptr;
  uint16_t* vcache = nullptr;
  uint32_t* flags = nullptr;       // hand-off counters of the loop kernel
  uint32_t* err_word = nullptr;
  int S_max = 0;
  int prefix_batch = 0;   // batch of the last fm_set_prefix (0 = none)
  std::vector<int> prefix_lens;   // per request, host copy of P_dev
  // batched tensor-core attention: TMA views of the q buffer and the K/V caches
  CUtensorMap tm_q{}, tm_k{}, tm_v{};
  bool tm_ok = false;
  int test_stall = 0;              // fm_test_stall: make the loop kernel's QKV hand-off unreachable
  long long test_spin = 0;         // fm_test_stall: wait budget in cycles (0: the default)
  std::map<std::pair<int, int>, cudaGraphExec_t> graphs;
  std::map<std::pair<int, int>, cudaGraph_t> graph_defs;
};

namespace {

fm_status set_err(fm_expert* h, fm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  if (h) h->err = buf;
  else g_create_error = buf;
  return s;
}

#define CK(call)                                                                          \
  do {                                                                                    \
    cudaError_t e_ = (call);                                                              \
    if (e_ != cudaSuccess)                                                                \
      return set_err(h, e_ == cudaErrorMemoryAllocation ? FM_ERR_OOM : FM_ERR_CUDA,       \
                     "%s: %s (%s:%d)", #call, cudaGetErrorString(e_), __FILE__, __LINE__); \
  } while (0)

template <class T>
fm_status dalloc(fm_expert* h, T** out, size_t bytes) {
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, bytes ? bytes : 16);
  if (e != cudaSuccess)
    return set_err(h, FM_ERR_OOM, "cudaMalloc(%zu bytes): %s", bytes, cudaGetErrorString(e));
  e = cudaMemset(p, 0, bytes ? bytes : 16);
  if (e != cudaSuccess) return set_err(h, FM_ERR_CUDA, "cudaMemset: %s", cudaGetErrorString(e));
  h->bufs.push_back({p, bytes});
  h->bytes += bytes;
  *out = static_cast<T*>(p);
  return FM_OK;
}
#define DALLOC(ptr, bytes)                        \
  do {                                            \
    fm_status s_ = dalloc(h, &(ptr), (bytes));    \
    if (s_ != FM_OK) return s_;                   \
  } while (0)

int round_up(int x, int m) { return (x + m - 1) / m * m; }

// `nseg` segments of `rows` rows of hd bf16 values as a 4-D TMA view
// (64 elements, hd/64 halves, rows, segments) with a (64, 1, 128, 1) box: one
// copy moves one 64-element half of 128 consecutive rows.  The driver's
// encoder is reached through the runtime (no link-time libcuda dependency).
bool encode_rows_map(CUtensorMap* m, void* base, int hd, int rows, int nseg) {
  typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  static EncodeFn fn = nullptr;
  if (fn == nullptr) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || f == nullptr) {
      cudaGetLastError();
      return false;
    }
    fn = reinterpret_cast<EncodeFn>(f);
  }
  const cuuint64_t dims[4] = {64, (cuuint64_t)(hd / 64), (cuuint64_t)rows, (cuuint64_t)nseg};
  const cuuint64_t strides[3] = {128, (cuuint64_t)hd * 2, (cuuint64_t)rows * hd * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Plans one linear over `nc` clusters (see GemmPlan).  Channels are dealt to
// clusters in units of NS x 16 so that per-cluster work differs by at most one
// unit; the K split starts at `max_ks` and is halved (more n-groups per
// cluster) until an n-group fits one MMA (N <= 256) and the work region
// (activation blocks + receive buffer).  `pair_cols`: owned columns come in
// gate/up pairs of even width (gate_up).
bool plan_gemm(GemmPlan& g, int N, int K, int nc, int max_ks, bool pair_cols) {
  if (K % 64 != 0 || nc < 1 || nc > kMaxClusters) return false;
  for (int ks = max_ks; ks >= 1; ks /= 2) {
    if ((K / 64) % ks != 0) continue;
    const int NS = kClusterSize / ks;
    // owners hold a multiple of 4 columns (16-byte partial pushes)
    const int unit = std::max(16, ks * 4);
    const int cunit = NS * unit;
    const int U = (N + cunit - 1) / cunit;
    const int q = U / nc, r = U % nc;
    g = GemmPlan{};
    g.N = N;
    g.K = K;
    g.KS = ks;
    g.NS = NS;
    g.kslice = K / ks;
    g.nchunk = g.kslice / 64;
    int off = 0;
    for (int c = 0; c < nc; ++c) {
      const int units = q + (c < r ? 1 : 0);
      g.ng[c] = units * unit;
      g.ch_off[c] = off;
      off += pair_cols ? NS * g.ng[c] / 2 : NS * g.ng[c];
      if (g.ng[c] > 0) g.busy_clusters++;
      g.max_ng = std::max(g.max_ng, g.ng[c]);
    }
    if (g.max_ng > 256) continue;
    // work region: activation blocks (later the outgoing partials), then the
    // receive buffer; the receive blocks have rows padded to 4 floats
    const size_t ownp = (size_t)((g.max_ng / ks + 3) & ~3);
    const size_t blocks = (size_t)ks * kRecvRows * ownp * 4;
    const size_t a_bytes = (size_t)g.nchunk * 8192;
    const size_t recv_off = ((a_bytes > blocks ? a_bytes : blocks) + 15) & ~(size_t)15;
    if (recv_off + blocks > (size_t)kWorkBytes) continue;
    return true;
  }
  return false;
}

// Source row (in the concatenated matrix of gemm g) of packed channel q of the
// n-group (cluster c, group grp); -1 for padding.
int source_row(const fm_expert* h, int g, int c, int grp, int q) {
  const fm_config& cf = h->cfg;
  const GemmPlan& gp = h->plan[g];
  const int ng = gp.ng[c];
  if (g == G_GU) {
    const int own = ng / gp.KS, uown = own / 2;
    const int ks = q / own, rr = q % own;
    const int u = gp.ch_off[c] + grp * (ng / 2) + ks * uown + (rr % uown);
    if (u >= cf.d_ff) return -1;
    return rr < uown ? u : cf.d_ff + u;
  }
  const int pc = gp.ch_off[c] + grp * ng + q;
  if (pc >= gp.N) return -1;
  if (g == G_QKV) {
    const int qn = cf.n_q_heads * cf.head_dim, kn = cf.n_kv_heads * cf.head_dim;
    if (pc < qn + kn) {
      // rotate-half partners (i, i + hd/2) are packed next to each other
      const int base = pc < qn ? 0 : qn;
      const int nn = pc - base;
      const int head = nn / cf.head_dim, w = nn % cf.head_dim;
      const int i = w >> 1;
      return base + head * cf.head_dim + i + (w & 1) * (cf.head_dim / 2);
    }
  }
  return pc;
}

fm_status build_plan(fm_expert* h) {
  const fm_config& c = h->cfg;
  const int nc = h->n_clusters;
  const int qkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  // QKV splits K at most 4 ways: its N per CTA then stays <= 128, where an
  // MMA costs the same as at half the width, and the split-K exchange halves
  if (!plan_gemm(h->plan[G_QKV], qkv, c.d_model, nc, 4, false) ||
      !plan_gemm(h->plan[G_O], c.d_model, c.n_q_heads * c.head_dim, nc, 8, false) ||
      !plan_gemm(h->plan[G_GU], 2 * c.d_ff, c.d_model, nc, 8, true) ||
      !plan_gemm(h->plan[G_DOWN], c.d_model, c.d_ff, nc, 8, false))
    return set_err(h, FM_ERR_UNSUPPORTED, "no work plan for this shape on %d clusters", nc);
  // epilogue work per compute thread: QKV rows per thread fit the 8 KB
  // rotation area at the end of the work region (8 rows x 128 threads); a
  // residual thread holds at most 4 column pairs in registers
  {
    const GemmPlan& pq = h->plan[G_QKV];
    const int npair_q = pq.max_ng / pq.KS / 2;
    const int per = npair_q > 0 ? 128 / npair_q : 0;
    const size_t ownp = (size_t)((pq.max_ng / pq.KS + 3) & ~3);
    const size_t blocks = (size_t)pq.KS * kRecvRows * ownp * 4;
    const size_t a_bytes = (size_t)pq.nchunk * 8192;
    const size_t recv_off = ((a_bytes > blocks ? a_bytes : blocks) + 15) & ~(size_t)15;
    if (per < 1 || (c.chunk_len + per - 1) / per > 8 || recv_off + blocks + 8192 > (size_t)kWorkBytes ||
        h->plan[G_O].max_ng / h->plan[G_O].KS > 16 || h->plan[G_DOWN].max_ng / h->plan[G_DOWN].KS > 16 ||
        h->plan[G_GU].max_ng / h->plan[G_GU].KS / 4 > 128)
      return set_err(h, FM_ERR_UNSUPPORTED, "too many owned columns per CTA on %d clusters", nc);
  }
  const int G = c.n_q_heads / c.n_kv_heads;
  h->att_blocks = (G * c.chunk_len + 63) / 64;
  h->q_rows = h->att_blocks * 64;
  // attention work region: q, K and V tiles and the combine buffer
  const size_t att = (size_t)3 * 64 * c.head_dim * 2 + (size_t)kClusterSize * 8 * (c.head_dim + 4) * 4;
  const size_t inproj = (size_t)c.chunk_len * c.action_dim * 4 +
                        (size_t)(h->plan[G_DOWN].max_ng / h->plan[G_DOWN].KS) * (c.action_dim + c.chunk_len) * 4;
  if (c.chunk_len * c.action_dim % 2 != 0 || (h->plan[G_DOWN].max_ng / h->plan[G_DOWN].KS) * c.action_dim > 32 * 128)
    return set_err(h, FM_ERR_UNSUPPORTED, "in-proj tile: chunk_len * action_dim must be even, owned rows x A <= 4096");
  if (att > (size_t)kWorkBytes || inproj > (size_t)kWorkBytes)
    return set_err(h, FM_ERR_UNSUPPORTED, "attention or in-proj tiles exceed shared memory");
  return FM_OK;
}

fm_status upload_rows(fm_expert* h, uint16_t* dst, const uint16_t* src, size_t elems, const char* what) {
  if (!src) return set_err(h, FM_ERR_INVALID_ARG, "weight %s is NULL", what);
  CK(cudaMemcpy(dst, src, elems * 2, cudaMemcpyDefault));
  return FM_OK;
}

// Index of packed channel q of n-group grp of cluster cl in a layer's scale
// table: the owners' columns in packing order (gate_up: 2 rows per u column).
int packed_index(const fm_expert* h, int g, int cl, int grp, int q) {
  const GemmPlan& gp = h->plan[g];
  return (g == G_GU ? 2 * gp.ch_off[cl] : gp.ch_off[cl]) + grp * gp.ng[cl] + q;
}

fm_status pack_weights(fm_expert* h, const fm_weights* w) {
  const fm_config& c = h->cfg;
  const int d = c.d_model, F = c.d_ff, qn = c.n_q_heads * c.head_dim,
            kn = c.n_kv_heads * c.head_dim;
  // quantised weights: E4M3 rows for every linear, or for all but gate_up,
  // whose rows are NVFP4 (64 codes + 4 block scales = 36 bytes)
  const bool nv4 = c.wtype == FM_W_FP8_NVFP4_GU;
  const bool w8a8 = c.wtype == FM_W_W8A8_E4M3;   // only the batched arena, in E4M3
  const bool fp8 = c.wtype == FM_W_FP8_E4M3 || nv4 || w8a8;
  auto fmt_of = [&](int g) { return !fp8 ? 0 : (nv4 && g == G_GU) ? 2 : 1; };
  auto row_bytes = [&](int g) -> uint64_t { const int f = fmt_of(g); return f == 0 ? 128 : f == 1 ? 64 : 36; };
  // Per-layer packing jobs (identical for every layer) and CTA spans.
  std::vector<PackChunk> jobs;
  std::vector<int32_t> rows;
  std::vector<uint32_t> span(h->n_ctas + 1, 0);
  uint64_t off = 0;
  for (int cta = 0; cta < h->n_ctas; ++cta) {
    span[cta] = (uint32_t)off;
    const int cl = cta / kClusterSize, rank = cta % kClusterSize;
    for (int g = 0; g < 4; ++g) {
      const GemmPlan& gp = h->plan[g];
      const int ng = gp.ng[cl];
      if (ng == 0) continue;
      const int grp = rank / gp.KS, ks = rank % gp.KS;
      const uint32_t roff = (uint32_t)rows.size();
      for (int q = 0; q < ng; ++q) rows.push_back(source_row(h, g, cl, grp, q));
      for (int i = 0; i < gp.nchunk; ++i) {
        PackChunk pc{};
        pc.dst_off = off;
        pc.rowidx_off = roff;
        pc.nrows = (uint16_t)ng;
        pc.mat = (uint8_t)g;
        pc.kb = (uint32_t)(ks * gp.nchunk + i);
        pc.fmt = (uint8_t)fmt_of(g);
        jobs.push_back(pc);
        off += (uint64_t)ng * row_bytes(g);
      }
    }
  }
  span[h->n_ctas] = (uint32_t)off;
  h->layer_bytes = off;
  if (off > 0xFFFFFFFFull) return set_err(h, FM_ERR_UNSUPPORTED, "layer span too large");
  // E4M3: packed-channel -> source-row map of each linear's scale table
  const int mrows[4] = {qn + 2 * kn, d, 2 * F, d};
  std::vector<int32_t> sc_src[4];
  if (fp8) {
    int at = 0;
    for (int g = 0; g < 4; ++g) {
      const GemmPlan& gp = h->plan[g];
      int n = 0;
      for (int cl = 0; cl < h->n_clusters; ++cl)
        if (gp.ng[cl] > 0) n = std::max(n, packed_index(h, g, cl, gp.NS - 1, gp.ng[cl] - 1) + 1);
      n = (n + 3) & ~3;
      sc_src[g].assign(n, -1);
      for (int cl = 0; cl < h->n_clusters; ++cl)
        for (int grp = 0; grp < gp.NS; ++grp)
          for (int q = 0; q < gp.ng[cl]; ++q) sc_src[g][packed_index(h, g, cl, grp, q)] = source_row(h, g, cl, grp, q);
      h->sc_off[g] = at;
      at += n;
    }
    h->sc_stride = at;
    h->pack_jobs = jobs;
    h->pack_rows = rows;
    h->row_scale.assign((size_t)c.n_layers * (mrows[0] + mrows[1] + mrows[2] + mrows[3]), 0.f);
    if (nv4) h->nv4_g.assign((size_t)2 * c.n_layers, 1.f);
    DALLOC(h->wscale, (size_t)c.n_layers * h->sc_stride * 4);
  }
  std::vector<float> sc_host(fp8 ? (size_t)c.n_layers * h->sc_stride : 0, 0.f);
  // Batched-path packing: each linear as [N/BN][K/64] chunks of BN rows
  // (gate_up tile j: gate rows 128 j .. then up rows 128 j ..); W8A8: E4M3
  // codes in [N/BN][K/128] chunks, same 128-byte rows.
  std::vector<PackChunk> bjobs;
  std::vector<int32_t> brows;
  if (h->batched) {
    const int Ns[4] = {qn + 2 * kn, d, 2 * F, d};
    const int Ks[4] = {d, qn, d, F};
    const int epi[4] = {BE_QKV, BE_RESID, BE_SWIGLU, BE_RESID};
    const int kcols = w8a8 ? 128 : 64;
    uint64_t boff = 0;
    for (int g = 0; g < 4; ++g) {
      const int bn = bgemm_bn(epi[g], Ns[g]), nkb = Ks[g] / kcols;
      h->boff[g] = boff;
      h->bw_off[g] = (int)brows.size();
      for (int nt = 0; nt < Ns[g] / bn; ++nt) {
        const uint32_t roff = (uint32_t)brows.size();
        for (int q = 0; q < bn; ++q) {
          int r = nt * bn + q;
          if (g == G_GU) r = q < bn / 2 ? nt * (bn / 2) + q : F + nt * (bn / 2) + (q - bn / 2);
          brows.push_back(r);
        }
        for (int kb = 0; kb < nkb; ++kb) {
          PackChunk pc{};
          pc.dst_off = boff + ((uint64_t)nt * nkb + kb) * bn * 128;
          pc.rowidx_off = roff;
          pc.nrows = (uint16_t)bn;
          pc.mat = (uint8_t)g;
          pc.kb = (uint32_t)kb;
          pc.fmt = (uint8_t)(w8a8 ? 1 : 0);
          bjobs.push_back(pc);
        }
      }
      boff += (uint64_t)Ns[g] * Ks[g] * (w8a8 ? 1 : 2);
    }
    h->blayer_bytes = boff;
    DALLOC(h->barena, (size_t)c.n_layers * boff);
    if (w8a8) {
      h->bw_stride = (int)brows.size();
      DALLOC(h->bwscale, (size_t)c.n_layers * h->bw_stride * 4);
      h->bpack_jobs = bjobs;
      h->bpack_rows = brows;
    }
  }
  std::vector<float> bw_host(w8a8 ? (size_t)c.n_layers * h->bw_stride : 0, 0.f);

  PackChunk* d_jobs = nullptr;
  int32_t* d_rows = nullptr;
  uint16_t** d_mats = nullptr;
  int* d_matk = nullptr;
  if (!w8a8) DALLOC(h->arena, (size_t)c.n_layers * off);
  DALLOC(h->span_off, span.size() * 4);
  CK(cudaMemcpy(h->span_off, span.data(), span.size() * 4, cudaMemcpyHostToDevice));
  // temporary buffers (freed at the end)
  void* tmp[9] = {};
  const size_t sz_qkv = (size_t)(qn + 2 * kn) * d, sz_o = (size_t)d * qn, sz_gu = (size_t)2 * F * d,
               sz_dn = (size_t)d * F;
  cudaError_t e = cudaSuccess;
  e = cudaMalloc(&tmp[0], sz_qkv * 2);
  if (e == cudaSuccess) e = cudaMalloc(&tmp[1], sz_o * 2);
  if (e == cudaSuccess) e = cudaMalloc(&tmp[2], sz_gu * 2);
  if (e == cudaSuccess) e = cudaMalloc(&tmp[3], sz_dn * 2);
  if (e == cudaSuccess) e = cudaMalloc(&tmp[4], jobs.size() * sizeof(PackChunk) + rows.size() * 4 + 64);
  if (e == cudaSuccess) e = cudaMalloc(&tmp[5], 8 * sizeof(void*) + 4 * sizeof(int));
  // E4M3: codes of the four linears and their row scales (NVFP4 gate_up:
  // one code per byte, then its block scales, two tensor scales, the amax word)
  if (e == cudaSuccess && fp8) e = cudaMalloc(&tmp[6], sz_qkv + sz_o + sz_gu + sz_dn + sz_gu / 16 + 64);
  if (e == cudaSuccess && fp8) e = cudaMalloc(&tmp[7], (size_t)(mrows[0] + mrows[1] + mrows[2] + mrows[3]) * 4);
  if (e == cudaSuccess && h->batched)
    e = cudaMalloc(&tmp[8], bjobs.size() * sizeof(PackChunk) + brows.size() * 4 + 64);
  PackChunk* d_bjobs = nullptr;
  int32_t* d_brows = nullptr;
  fm_status st = FM_OK;
  if (e != cudaSuccess) {
    st = set_err(h, FM_ERR_OOM, "packing buffers: %s", cudaGetErrorString(e));
  } else {
    d_jobs = static_cast<PackChunk*>(tmp[4]);
    d_rows = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(tmp[4]) + jobs.size() * sizeof(PackChunk));
    d_mats = static_cast<uint16_t**>(tmp[5]);
    d_matk = reinterpret_cast<int*>(static_cast<uint8_t*>(tmp[5]) + 8 * sizeof(void*));
    uint16_t* mats[4] = {static_cast<uint16_t*>(tmp[0]), static_cast<uint16_t*>(tmp[1]),
                         static_cast<uint16_t*>(tmp[2]), static_cast<uint16_t*>(tmp[3])};
    const int matk[4] = {d, qn, d, F};
    uint8_t* q8[4] = {};
    float* rs[4] = {};
    uint8_t* sb4 = nullptr;     // NVFP4 gate_up block scales [2F][d/16]
    float* g4 = nullptr;        // [2]: gate, up tensor scales
    unsigned int* amax4 = nullptr;
    if (fp8) {
      q8[0] = static_cast<uint8_t*>(tmp[6]);
      q8[1] = q8[0] + sz_qkv;
      q8[2] = q8[1] + sz_o;
      q8[3] = q8[2] + sz_gu;
      sb4 = q8[3] + sz_dn;
      g4 = reinterpret_cast<float*>(sb4 + sz_gu / 16 + 16 - (sz_gu / 16) % 16);
      amax4 = reinterpret_cast<unsigned int*>(g4 + 4);
      rs[0] = static_cast<float*>(tmp[7]);
      for (int g = 1; g < 4; ++g) rs[g] = rs[g - 1] + mrows[g - 1];
    }
    e = cudaMemcpy(d_jobs, jobs.data(), jobs.size() * sizeof(PackChunk), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d_rows, rows.data(), rows.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && h->batched) {
      d_bjobs = static_cast<PackChunk*>(tmp[8]);
      d_brows = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(tmp[8]) + bjobs.size() * sizeof(PackChunk));
      e = cudaMemcpy(d_bjobs, bjobs.data(), bjobs.size() * sizeof(PackChunk), cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(d_brows, brows.data(), brows.size() * 4, cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && fp8) e = cudaMemcpy(d_mats, q8, sizeof(q8), cudaMemcpyHostToDevice);
    else if (e == cudaSuccess) e = cudaMemcpy(d_mats, mats, sizeof(mats), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d_matk, matk, sizeof(matk), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) st = set_err(h, FM_ERR_CUDA, "pack tables: %s", cudaGetErrorString(e));
    for (int l = 0; l < c.n_layers && st == FM_OK; ++l) {
      const fm_layer_weights& lw = w->layers[l];
      if (!lw.wq || !lw.wk || !lw.wv || !lw.wo || !lw.w_gate || !lw.w_up || !lw.w_down) {
        st = set_err(h, FM_ERR_INVALID_ARG, "layer %d has a NULL weight", l);
        break;
      }
      e = cudaMemcpy(mats[0], lw.wq, (size_t)qn * d * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[0] + (size_t)qn * d, lw.wk, (size_t)kn * d * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[0] + (size_t)(qn + kn) * d, lw.wv, (size_t)kn * d * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[1], lw.wo, sz_o * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[2], lw.w_gate, (size_t)F * d * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[2] + (size_t)F * d, lw.w_up, (size_t)F * d * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mats[3], lw.w_down, sz_dn * 2, cudaMemcpyDefault);
      if (fp8) {
        // R8: per-row absmax / 448 and E4M3 codes of every linear, then the
        // codes go into the arena and the scales into the packed-order table
        for (int g = 0; g < 4 && e == cudaSuccess; ++g) e = launch_fp8_quantize(mats[g], mrows[g], matk[g], rs[g], q8[g], 0);
        if (e == cudaSuccess && nv4) {
          // R10 for gate and up separately (their own tensor scales), over the
          // E4M3 codes of gate_up, which only the scale table below still reads
          for (int t = 0; t < 2 && e == cudaSuccess; ++t)
            e = launch_nvfp4_quantize(mats[G_GU] + (size_t)t * F * d, F, d, amax4, q8[G_GU] + (size_t)t * F * d,
                                      sb4 + (size_t)t * F * (d / 16), g4 + t, 0);
        }
        if (e == cudaSuccess && !w8a8)
          e = launch_pack8(d_jobs, (int)jobs.size(), d_rows, reinterpret_cast<const uint8_t* const*>(d_mats), d_matk,
                           h->arena + (size_t)l * off, 0);
        if (e == cudaSuccess && w8a8)
          e = launch_pack8_tile(d_bjobs, (int)bjobs.size(), d_brows, reinterpret_cast<const uint8_t* const*>(d_mats),
                                d_matk, h->barena + (size_t)l * h->blayer_bytes, 0);
        if (e == cudaSuccess && nv4)
          e = launch_pack_nvfp4(d_jobs, (int)jobs.size(), d_rows, q8[G_GU], sb4, d, h->arena + (size_t)l * off, 0);
        float gh[2] = {1.f, 1.f};
        if (e == cudaSuccess && nv4) e = cudaMemcpy(gh, g4, 8, cudaMemcpyDeviceToHost);
        if (e == cudaSuccess && nv4) {
          h->nv4_g[2 * l] = gh[0];
          h->nv4_g[2 * l + 1] = gh[1];
        }
        float* lrs = h->row_scale.data() + (size_t)l * (mrows[0] + mrows[1] + mrows[2] + mrows[3]);
        if (e == cudaSuccess)
          e = cudaMemcpy(lrs, rs[0], (size_t)(mrows[0] + mrows[1] + mrows[2] + mrows[3]) * 4, cudaMemcpyDeviceToHost);
        if (e == cudaSuccess && w8a8) {
          // GEMM column i of linear g holds source row brows[i] of that linear
          int rbase = 0;
          for (int g = 0; g < 4; ++g) {
            const int end = g < 3 ? h->bw_off[g + 1] : h->bw_stride;
            for (int i = h->bw_off[g]; i < end; ++i)
              bw_host[(size_t)l * h->bw_stride + i] = lrs[rbase + brows[i]];
            rbase += mrows[g];
          }
        }
        if (e == cudaSuccess) {
          const float* src = lrs;
          for (int g = 0; g < 4; ++g) {
            float* dst = sc_host.data() + (size_t)l * h->sc_stride + h->sc_off[g];
            for (size_t i = 0; i < sc_src[g].size(); ++i) {
              const int sr = sc_src[g][i];
              // NVFP4 gate_up columns carry their tensor's scale (gate rows, then up rows)
              dst[i] = sr < 0 ? 0.f : (nv4 && g == G_GU) ? h->nv4_g[2 * l + (sr < F ? 0 : 1)] : src[sr];
            }
            src += mrows[g];
          }
        }
      } else if (e == cudaSuccess) {
        e = launch_pack(d_jobs, (int)jobs.size(), d_rows, d_mats, d_matk, h->arena + (size_t)l * off, 0);
        if (e == cudaSuccess && h->batched)
          e = launch_pack(d_bjobs, (int)bjobs.size(), d_brows, d_mats, d_matk,
                          h->barena + (size_t)l * h->blayer_bytes, 0);
      }
      if (e == cudaSuccess) e = cudaDeviceSynchronize();
      if (e != cudaSuccess) st = set_err(h, FM_ERR_CUDA, "packing layer %d: %s", l, cudaGetErrorString(e));
    }
    if (st == FM_OK && fp8) {
      e = cudaMemcpy(h->wscale, sc_host.data(), sc_host.size() * 4, cudaMemcpyHostToDevice);
      if (e == cudaSuccess && w8a8) e = cudaMemcpy(h->bwscale, bw_host.data(), bw_host.size() * 4, cudaMemcpyHostToDevice);
      if (e != cudaSuccess) st = set_err(h, FM_ERR_CUDA, "scale table: %s", cudaGetErrorString(e));
    }
  }
  for (void* p : tmp)
    if (p) cudaFree(p);
  if (st != FM_OK) return st;

  // Time MLP: W1 plain bf16, W2 packed in tiles of 128 rows x 64 columns.
  DALLOC(h->w1, (size_t)d * kTimeDim * 2);
  st = upload_rows(h, h->w1, w->time_w1, (size_t)d * kTimeDim, "time_w1");
  if (st != FM_OK) return st;
  const int n_mod = h->n_mod;
  const int ntiles = (n_mod + 127) / 128, nkb = d / 64;
  DALLOC(h->w2_packed, (size_t)ntiles * nkb * 16384);
  {
    std::vector<PackChunk> tj;
    std::vector<int32_t> tr((size_t)ntiles * 128);
    for (int t = 0; t < ntiles; ++t) {
      for (int q = 0; q < 128; ++q) tr[(size_t)t * 128 + q] = (t * 128 + q < n_mod) ? t * 128 + q : -1;
      for (int kb = 0; kb < nkb; ++kb) {
        PackChunk pc{};
        pc.dst_off = ((uint64_t)t * nkb + kb) * 16384;
        pc.rowidx_off = (uint32_t)t * 128;
        pc.nrows = 128;
        pc.mat = 0;
        pc.kb = (uint32_t)kb;
        tj.push_back(pc);
      }
    }
    void* t2 = nullptr;
    void* tt = nullptr;
    e = cudaMalloc(&t2, (size_t)n_mod * d * 2);
    if (e == cudaSuccess) e = cudaMalloc(&tt, tj.size() * sizeof(PackChunk) + tr.size() * 4 + 64);
    if (e != cudaSuccess) {
      if (t2) cudaFree(t2);
      return set_err(h, FM_ERR_OOM, "time_w2 staging: %s", cudaGetErrorString(e));
    }
    PackChunk* dj = static_cast<PackChunk*>(tt);
    int32_t* dr = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(tt) + tj.size() * sizeof(PackChunk));
    // reuse a small device table for the matrix pointer / width
    void* tm = nullptr;
    e = cudaMalloc(&tm, sizeof(void*) + sizeof(int));
    if (e == cudaSuccess) {
      uint16_t* mp = static_cast<uint16_t*>(t2);
      int kk = d;
      e = cudaMemcpy(tm, &mp, sizeof(void*), cudaMemcpyHostToDevice);
      if (e == cudaSuccess) e = cudaMemcpy(static_cast<uint8_t*>(tm) + sizeof(void*), &kk, sizeof(int), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess && !w->time_w2) e = cudaErrorInvalidValue;
    if (e == cudaSuccess) e = cudaMemcpy(t2, w->time_w2, (size_t)n_mod * d * 2, cudaMemcpyDefault);
    if (e == cudaSuccess) e = cudaMemcpy(dj, tj.data(), tj.size() * sizeof(PackChunk), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(dr, tr.data(), tr.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = launch_pack(dj, (int)tj.size(), dr, static_cast<uint16_t* const*>(tm),
                      reinterpret_cast<const int*>(static_cast<uint8_t*>(tm) + sizeof(void*)), h->w2_packed, 0);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    cudaFree(t2);
    cudaFree(tt);
    if (tm) cudaFree(tm);
    if (e != cudaSuccess) return set_err(h, FM_ERR_CUDA, "packing time_w2: %s", cudaGetErrorString(e));
  }
  DALLOC(h->w_in, (size_t)d * c.action_dim * 2);
  st = upload_rows(h, h->w_in, w->in_proj, (size_t)d * c.action_dim, "in_proj");
  if (st != FM_OK) return st;
  if (h->batched) {
    DALLOC(h->w_in_t, (size_t)d * c.action_dim * 2);
    CK(launch_transpose_bf16(h->w_in, d, c.action_dim, h->w_in_t, 0));
    CK(cudaDeviceSynchronize());
  }
  DALLOC(h->w_out, (size_t)d * c.action_dim * 2);
  st = upload_rows(h, h->w_out, w->out_proj, (size_t)d * c.action_dim, "out_proj");
  if (st != FM_OK) return st;
  if (w->out_bias) {
    DALLOC(h->out_bias, (size_t)c.action_dim * 4);
    CK(cudaMemcpy(h->out_bias, w->out_bias, (size_t)c.action_dim * 4, cudaMemcpyDefault));
  }
  return FM_OK;
}

// The batched path needs whole 128-column weight tiles, the in-proj's
// 256-column thread mapping and at most 1024 residual columns.
bool batched_shape_ok(const fm_config& c) {
  const int qkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim;
  return c.d_model % 256 == 0 && c.d_model <= 1024 && c.d_ff % 128 == 0 && qkv % 128 == 0 &&
         (c.n_q_heads * c.head_dim) % 64 == 0 && (c.head_dim == 64 || c.head_dim == 128);
}

// W8A8 runs every batch on the batched path and also quantises o and u per
// row (K a multiple of 256, at most 4096).
bool w8a8_shape_ok(const fm_config& c) {
  const int qn = c.n_q_heads * c.head_dim;
  return batched_shape_ok(c) && qn % 256 == 0 && qn <= 4096 && c.d_ff % 256 == 0 && c.d_ff <= 4096;
}

fm_status check_config(const fm_config* c) {
  fm_expert* h = nullptr;
  if (!c) return set_err(h, FM_ERR_INVALID_ARG, "config is NULL");
  if (c->n_layers < 1 || c->d_model < 64 || c->n_q_heads < 1 || c->n_kv_heads < 1 ||
      c->d_ff < 64 || c->action_dim < 1 || c->chunk_len < 1 || c->max_prefix < 0 ||
      c->max_batch < 1 || c->max_steps < 1)
    return set_err(h, FM_ERR_INVALID_ARG, "non-positive size in config");
  if (c->d_model % 64 || c->d_ff % 64 || (c->n_q_heads * c->head_dim) % 64)
    return set_err(h, FM_ERR_INVALID_ARG, "d_model, d_ff and n_q_heads*head_dim must be multiples of 64");
  if (c->head_dim != 64 && c->head_dim != 128)
    return set_err(h, FM_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (c->n_q_heads % c->n_kv_heads)
    return set_err(h, FM_ERR_INVALID_ARG, "n_q_heads must be a multiple of n_kv_heads");
  if (c->chunk_len > kMaxT) return set_err(h, FM_ERR_UNSUPPORTED, "chunk_len must be <= %d", kMaxT);
  if (c->action_dim > 128) return set_err(h, FM_ERR_UNSUPPORTED, "action_dim must be <= 128");
  if (c->d_model > 1024) return set_err(h, FM_ERR_UNSUPPORTED, "d_model must be <= 1024");
  if (c->max_steps > kRows) return set_err(h, FM_ERR_INVALID_ARG, "max_steps must be <= %d", kRows);
  if (!(c->rms_eps > 0.f) || !(c->rope_base > 0.f))
    return set_err(h, FM_ERR_INVALID_ARG, "rms_eps and rope_base must be positive");
  if (c->wtype != FM_W_BF16 && c->wtype != FM_W_FP8_E4M3 && c->wtype != FM_W_FP8_NVFP4_GU &&
      c->wtype != FM_W_W8A8_E4M3)
    return set_err(h, FM_ERR_INVALID_ARG, "unknown wtype %d", c->wtype);
  if (c->wtype == FM_W_W8A8_E4M3 && !w8a8_shape_ok(*c))
    return set_err(h, FM_ERR_UNSUPPORTED,
                   "W8A8 needs d_model a multiple of 256 (<= 1024), n_q_heads*head_dim and d_ff multiples of 256 "
                   "(<= 4096), (n_q_heads + 2 n_kv_heads)*head_dim a multiple of 128");
  return FM_OK;
}

void free_all(fm_expert* h) {
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  for (auto& kv : h->graph_defs) cudaGraphDestroy(kv.second);
  h->graphs.clear();
  h->graph_defs.clear();
  for (auto& b : h->bufs) cudaFree(b.p);
  h->bufs.clear();
  if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
  h->cap_stream = nullptr;
}

bool is_device_ptr(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

StepParams base_params(const fm_expert* h) {
  const fm_config& c = h->cfg;
  StepParams p{};
  p.L = c.n_layers;
  p.d = c.d_model;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.hd = c.head_dim;
  p.F = c.d_ff;
  p.A = c.action_dim;
  p.T = c.chunk_len;
  p.S_max = h->S_max;
  p.B_cap = c.max_batch;
  p.b = 0;
  p.P_dev = h->P_dev;
  p.eps = c.rms_eps;
  p.n_clusters = h->n_clusters;
  p.n_ctas = h->n_ctas;
  for (int g = 0; g < 4; ++g) p.g[g] = h->plan[g];
  p.att_blocks = h->att_blocks;
  p.q_rows = h->q_rows;
  p.arena = h->arena;
  p.layer_bytes = h->layer_bytes;
  p.span_off = h->span_off;
  p.w_in = h->w_in;
  p.w_out = h->w_out;
  p.out_bias = h->out_bias;
  p.mod = h->mod;
  p.n_mod = h->n_mod;
  p.rope = h->rope;
  p.x = h->x;
  p.vbuf = h->vbuf;
  p.h_a = h->h_a;
  p.h_b = h->h_b;
  p.z_a = h->z_a;
  p.z_f = h->z_f;
  p.o_act = h->o_act;
  p.u_act = h->u_act;
  p.sumsq_a = h->sumsq_a;
  p.sumsq_f = h->sumsq_f;
  p.qbuf = h->qbuf;
  p.kcache = h->kcache;
  p.vcache = h->vcache;
  p.flags = h->flags;
  p.err = h->err_word;
  for (int g = 0; g < 4; ++g)
    p.wfmt[g] = c.wtype == FM_W_BF16 ? 0 : (c.wtype == FM_W_FP8_NVFP4_GU && g == G_GU) ? 2 : 1;
  p.wscale = h->wscale;
  p.sc_stride = h->sc_stride;
  for (int g = 0; g < 4; ++g) p.sc_off[g] = h->sc_off[g];
  p.step0 = 0;
  p.step1 = 0;
  p.layer0 = 0;
  p.layer1 = c.n_layers;
  {
    const GemmPlan &go = h->plan[G_O], &gd = h->plan[G_DOWN];
    bool same = go.KS == gd.KS;
    for (int i = 0; i < kMaxClusters && same; ++i) same = go.ng[i] == gd.ng[i] && go.ch_off[i] == gd.ch_off[i];
    p.h_regs = same ? 1 : 0;
  }
  p.store_mid = 0;
  p.do_inproj = 1;
  p.do_outproj = 1;
  p.update_x = 1;
  p.dt = 0.f;
  p.spin_budget = h->test_spin > 0 ? h->test_spin : 4000000000LL;   // ~2 s at 2 GHz
  p.stall_test = h->test_stall;
  p.tlog = nullptr;
  p.tlog_stride = 0;
  p.tlog_mma_off = 0;
  p.tlog_chunk_off = 0;
  p.tlog_chunks = 0;
  return p;
}

TimeParams time_params(const fm_expert* h, int steps) {
  TimeParams t{};
  t.n_steps = steps;
  t.d = h->cfg.d_model;
  t.n_mod = h->n_mod;
  t.w1 = h->w1;
  t.w2_packed = h->w2_packed;
  t.h1_act = h->h1_act;
  t.mod = h->mod;
  t.err = h->err_word;
  t.spin_budget = 4000000000LL;
  return t;
}

// Batched path: Euler steps step0 .. step1 - 1 of a `steps`-step schedule for
// `batch` requests together (x in h->x, velocities to h->vbuf; x updated when
// `update`).  The modulation rows must already be in h->mod.
// `hook` (test hook, null on the product path) runs on the host after each
// stage: (l, 0) layer l's attention norm is in bz_a and its input in bh;
// (l, 1) q and the chunk's K/V rows; (l, 2) attention output; (l, 3) h after
// o_proj; (l, 4) FFN norm; (l, 5) SwiGLU output; (l, 6) h after down;
// (L, 7) the velocity.
using BatchHook = std::function<cudaError_t(int, int)>;

cudaError_t enqueue_batched(fm_expert* h, int batch, int step0, int step1, int steps, bool update,
                            cudaStream_t st, const BatchHook* hook = nullptr) {
  const fm_config& c = h->cfg;
  const int T = c.chunk_len, d = c.d_model, M = batch * T, L = c.n_layers;
  const int qn = c.n_q_heads * c.head_dim, kn = c.n_kv_heads * c.head_dim, F = c.d_ff;
  const int Mp = (M + kBM - 1) / kBM * kBM;
  const size_t lay = (size_t)c.max_batch * c.n_kv_heads * h->S_max * c.head_dim;
  BRowParams r{};
  r.M = M;
  r.T = T;
  r.A = c.action_dim;
  r.d = d;
  r.eps = c.rms_eps;
  r.dt = -1.0f / (float)steps;
  r.x = h->x;
  r.x_out = update ? h->x : nullptr;
  r.v_out = h->vbuf;
  r.w_in_t = h->w_in_t;
  r.w_out = h->w_out;
  r.out_bias = h->out_bias;
  r.h = h->bh;
  BGemmParams g{};
  g.M = M;
  g.Mp = Mp;
  g.h = h->bh;   // the residual GEMMs add their branch into h
  g.u_act = h->bu;
  g.F = F;
  g.qbuf = h->bq;
  g.rope = h->rope;
  g.rope_stride_b = T;
  g.P_dev = h->P_dev;
  g.T = T;
  g.Hq = c.n_q_heads;
  g.Hkv = c.n_kv_heads;
  g.hd = c.head_dim;
  g.S_max = h->S_max;
  g.q_rows = h->q_rows;
  g.err = h->err_word;
  g.spin_budget = 4000000000LL;
  // W8A8: row scales of the four GEMM inputs; o and u are quantised by a
  // row pass after the kernels that write them in bf16
  const size_t Mcap = (size_t)h->Mp;
  float* sa_za = h->w8a8 ? h->bsa : nullptr;
  float* sa_o = h->w8a8 ? h->bsa + Mcap : nullptr;
  float* sa_zf = h->w8a8 ? h->bsa + 2 * Mcap : nullptr;
  float* sa_u = h->w8a8 ? h->bsa + 3 * Mcap : nullptr;
  BQuantParams qo{h->bo, h->bo8, sa_o, M, qn};
  BQuantParams qu{h->bu, h->bu8, sa_u, M, F};
  BAttnParams a{};
  a.tm_q = h->tm_q;
  a.tm_k = h->tm_k;
  a.tm_v = h->tm_v;
  a.qbuf = h->bq;
  a.o_act = h->bo;
  a.P_dev = h->P_dev;
  a.B = batch;
  a.T = T;
  a.Hq = c.n_q_heads;
  a.Hkv = c.n_kv_heads;
  a.hd = c.head_dim;
  a.S_max = h->S_max;
  a.q_rows = h->q_rows;
  a.qblocks = (c.n_q_heads / c.n_kv_heads * T + 63) / 64;
  a.err = h->err_word;
  a.spin_budget = 4000000000LL;
  cudaError_t e = cudaSuccess;
  for (int s = step0; s < step1 && e == cudaSuccess; ++s) {
    const float* mrow = h->mod + (size_t)s * h->n_mod;
    r.s = mrow;
    r.b = mrow + d;
    r.z = h->bz_a;
    r.zs = sa_za;
    e = launch_binproj(r, st);
    if (e == cudaSuccess) e = launch_bresnorm(r, st);   // layer 0's attention norm
    auto stage = [&](int l, int k) {
      if (hook != nullptr && e == cudaSuccess) e = (*hook)(l, k);
    };
    for (int l = 0; l < L && e == cudaSuccess; ++l) {
      stage(l, 0);
      const float* lm = mrow + (size_t)6 * l * d;
      const uint8_t* wl = h->barena + (size_t)l * h->blayer_bytes;
      const float* bws = h->w8a8 ? h->bwscale + (size_t)l * h->bw_stride : nullptr;
      auto wsc = [&](int gi) { return bws != nullptr ? bws + h->bw_off[gi] : nullptr; };
      // QKV + RoPE -> q, cache rows P .. P + T - 1
      g.A = reinterpret_cast<const uint8_t*>(h->bz_a);
      g.a_scale = sa_za;
      g.w_scale = wsc(G_QKV);
      g.W = wl + h->boff[G_QKV];
      g.K = d;
      g.N = qn + 2 * kn;
      g.kc = h->kcache + l * lay;
      g.vc = h->vcache + l * lay;
      e = launch_bgemm(g, BE_QKV, h->n_sms, st);
      stage(l, 1);
      a.kc = h->kcache + l * lay;
      a.vc = h->vcache + l * lay;
      a.seg_base = l * c.max_batch * c.n_kv_heads;
      if (e == cudaSuccess) e = h->tm_ok ? launch_battn_tc(a, st) : launch_battn(a, st);
      if (e == cudaSuccess && h->w8a8) e = launch_browquant(qo, st);
      stage(l, 2);
      // o_proj + gated residual, then the FFN norm
      g.A = h->w8a8 ? h->bo8 : reinterpret_cast<const uint8_t*>(h->bo);
      g.a_scale = sa_o;
      g.w_scale = wsc(G_O);
      g.W = wl + h->boff[G_O];
      g.K = qn;
      g.N = d;
      g.gate = lm + 2 * d;
      if (e == cudaSuccess) e = launch_bgemm(g, BE_RESID, h->n_sms, st);
      stage(l, 3);
      r.s = lm + 3 * d;
      r.b = lm + 4 * d;
      r.z = h->bz_f;
      r.zs = sa_zf;
      if (e == cudaSuccess) e = launch_bresnorm(r, st);
      stage(l, 4);
      // gate_up + SwiGLU, down + gated residual
      g.A = reinterpret_cast<const uint8_t*>(h->bz_f);
      g.a_scale = sa_zf;
      g.w_scale = wsc(G_GU);
      g.W = wl + h->boff[G_GU];
      g.K = d;
      g.N = 2 * F;
      if (e == cudaSuccess) e = launch_bgemm(g, BE_SWIGLU, h->n_sms, st);
      if (e == cudaSuccess && h->w8a8) e = launch_browquant(qu, st);
      stage(l, 5);
      g.A = h->w8a8 ? h->bu8 : reinterpret_cast<const uint8_t*>(h->bu);
      g.a_scale = sa_u;
      g.w_scale = wsc(G_DOWN);
      g.W = wl + h->boff[G_DOWN];
      g.K = F;
      g.N = d;
      g.gate = lm + 5 * d;
      if (e == cudaSuccess) e = launch_bgemm(g, BE_RESID, h->n_sms, st);
      stage(l, 6);
      // the next layer's attention norm (none after the last layer: the
      // out-proj kernel applies the final norm)
      r.s = lm + 6 * d;
      r.b = lm + 7 * d;
      r.z = h->bz_a;
      r.zs = sa_za;
      if (e == cudaSuccess && l + 1 < L) e = launch_bresnorm(r, st);
    }
    r.s = mrow + (size_t)6 * L * d;
    r.b = r.s + d;
    if (e == cudaSuccess) e = launch_boutproj(r, st);
    stage(L, 7);
  }
  return e;
}

// Whether `batch` requests run on the batched path: B >= 2 on a handle that
// has it, every B on a W8A8 handle.
bool use_batched(const fm_expert* h, int batch) { return h->batched && (batch >= 2 || h->w8a8); }

// Enqueues one full denoise of `batch` requests (x already in h->x).
cudaError_t enqueue_denoise(fm_expert* h, int batch, int steps, cudaStream_t st) {
  if (use_batched(h, batch)) {
    cudaError_t e = launch_time(time_params(h, steps), h->n_sms, st);
    if (e != cudaSuccess) return e;
    return enqueue_batched(h, batch, 0, steps, steps, true, st);
  }
  cudaError_t e = cudaMemsetAsync(h->flags, 0, kFlagBytes, st);
  if (e != cudaSuccess) return e;
  e = launch_time(time_params(h, steps), h->n_sms, st);
  if (e != cudaSuccess) return e;
  const size_t xs = (size_t)h->cfg.chunk_len * h->cfg.action_dim;
  for (int b = 0; b < batch; ++b) {
    StepParams p = base_params(h);
    p.b = b;
    p.x = h->x + b * xs;
    p.vbuf = h->vbuf + b * xs;
    p.step0 = 0;
    p.step1 = steps;
    p.dt = -1.0f / (float)steps;
    if (b > 0) {
      e = cudaMemsetAsync(h->flags, 0, kFlagBytes, st);
      if (e != cudaSuccess) return e;
    }
    e = launch_step(p, st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

fm_status check_err_word(fm_expert* h) {
  uint32_t w = 0;
  CK(cudaMemcpy(&w, h->err_word, 4, cudaMemcpyDeviceToHost));
  if (w) {
    CK(cudaMemset(h->err_word, 0, 4));
    return set_err(h, FM_ERR_TIMEOUT, "a device-side wait gave up (code 0x%x)", w);
  }
  return FM_OK;
}

}  // namespace

extern "C" {
#pragma GCC visibility push(default)

int fm_abi_version(void) { return FM_ABI_VERSION; }

const char* fm_status_string(fm_status s) {
  switch (s) {
    case FM_OK: return "FM_OK";
    case FM_ERR_INVALID_ARG: return "FM_ERR_INVALID_ARG";
    case FM_ERR_NOT_READY: return "FM_ERR_NOT_READY";
    case FM_ERR_OOM: return "FM_ERR_OOM";
    case FM_ERR_CUDA: return "FM_ERR_CUDA";
    case FM_ERR_TIMEOUT: return "FM_ERR_TIMEOUT";
    case FM_ERR_UNSUPPORTED: return "FM_ERR_UNSUPPORTED";
  }
  return "unknown fm_status";
}

const char* fm_last_error(const fm_expert* h) {
  return h ? h->err.c_str() : g_create_error.c_str();
}

fm_status fm_expert_create(const fm_config* cfg, const fm_weights* w, int device, fm_expert** out) {
  fm_expert* h = nullptr;
  g_create_error.clear();
  if (!out) return set_err(h, FM_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  fm_status st = check_config(cfg);
  if (st != FM_OK) return st;
  if (!w || !w->layers || !w->time_w1 || !w->time_w2 || !w->in_proj || !w->out_proj)
    return set_err(h, FM_ERR_INVALID_ARG, "weights or a weight pointer is NULL");
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return set_err(h, FM_ERR_UNSUPPORTED, "no CUDA device");
  }
  if (device < 0 || device >= ndev) return set_err(h, FM_ERR_INVALID_ARG, "device %d out of range", device);
  cudaDeviceProp prop{};
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess)
    return set_err(h, FM_ERR_CUDA, "cudaGetDeviceProperties failed");
  if (prop.major != 10 || prop.minor != 0)
    return set_err(h, FM_ERR_UNSUPPORTED, "device %d is sm_%d%d; the library is compiled for sm_100a", device,
                   prop.major, prop.minor);
  if (cudaSetDevice(device) != cudaSuccess) return set_err(h, FM_ERR_CUDA, "cudaSetDevice failed");

  h = new fm_expert();
  h->cfg = *cfg;
  h->device = device;
  h->n_sms = prop.multiProcessorCount;
  const fm_config& c = h->cfg;
  h->n_mod = c.n_layers * 6 * c.d_model + 2 * c.d_model;
  h->S_max = c.max_prefix + c.chunk_len;
  auto bail = [&](fm_status s) {
    g_create_error = h->err;
    free_all(h);
    delete h;
    return s;
  };
  int ncl = 0;
  if (step_max_clusters(&ncl) != cudaSuccess || ncl < 1) {
    cudaGetLastError();
    set_err(h, FM_ERR_UNSUPPORTED, "no co-resident clusters of %d CTAs", kClusterSize);
    return bail(FM_ERR_UNSUPPORTED);
  }
  h->n_clusters = std::min(std::min(ncl, h->n_sms / kClusterSize), kMaxClusters);
  h->n_ctas = h->n_clusters * kClusterSize;
  if ((st = build_plan(h)) != FM_OK) return bail(st);
  if (cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    set_err(h, FM_ERR_CUDA, "stream creation failed");
    return bail(FM_ERR_CUDA);
  }
  // the batched path: bf16 handles with max_batch >= 2, and every W8A8 handle
  // (its shapes were checked with the config)
  h->w8a8 = c.wtype == FM_W_W8A8_E4M3;
  h->batched = batched_shape_ok(c) && ((c.wtype == FM_W_BF16 && c.max_batch >= 2) || h->w8a8);
  if ((st = pack_weights(h, w)) != FM_OK) return bail(st);

  const size_t T = c.chunk_len, A = c.action_dim, d = c.d_model;
  const size_t B = c.max_batch;
#define ALLOC_OR_BAIL(ptr, bytes)                           \
  do {                                                      \
    fm_status s_ = dalloc(h, &(ptr), (bytes));              \
    if (s_ != FM_OK) return bail(s_);                       \
  } while (0)
  ALLOC_OR_BAIL(h->mod, (size_t)c.max_steps * h->n_mod * 4);
  ALLOC_OR_BAIL(h->h1_act, (size_t)kRows * d * 2);
  ALLOC_OR_BAIL(h->rope, B * T * c.head_dim * 4);
  ALLOC_OR_BAIL(h->P_dev, B * 4);
  ALLOC_OR_BAIL(h->x, B * T * A * 4);
  ALLOC_OR_BAIL(h->vbuf, B * T * A * 4);
  ALLOC_OR_BAIL(h->h_a, T * d * 4);
  ALLOC_OR_BAIL(h->h_b, T * d * 4);
  ALLOC_OR_BAIL(h->z_a, (size_t)2 * kRows * d * 2);
  ALLOC_OR_BAIL(h->z_f, (size_t)2 * kRows * d * 2);
  ALLOC_OR_BAIL(h->o_act, (size_t)2 * kRows * c.n_q_heads * c.head_dim * 2);
  ALLOC_OR_BAIL(h->u_act, (size_t)2 * kRows * c.d_ff * 2);
  ALLOC_OR_BAIL(h->sumsq_a, (size_t)h->n_ctas * kRows * 4);
  ALLOC_OR_BAIL(h->sumsq_f, (size_t)h->n_ctas * kRows * 4);
  ALLOC_OR_BAIL(h->qbuf, (size_t)c.n_kv_heads * h->q_rows * c.head_dim * 2);
  const size_t kv = (size_t)c.n_layers * B * c.n_kv_heads * h->S_max * c.head_dim * 2;
  ALLOC_OR_BAIL(h->kcache, kv);
  ALLOC_OR_BAIL(h->vcache, kv);
  ALLOC_OR_BAIL(h->flags, kFlagBytes);
  ALLOC_OR_BAIL(h->err_word, 4);
  if (h->batched) {
    h->Mp = (int)((B * T + kBM - 1) / kBM * kBM);
    const size_t Mp = (size_t)h->Mp;
    ALLOC_OR_BAIL(h->bz_a, Mp * d * 2);
    ALLOC_OR_BAIL(h->bz_f, Mp * d * 2);
    ALLOC_OR_BAIL(h->bo, Mp * c.n_q_heads * c.head_dim * 2);
    ALLOC_OR_BAIL(h->bu, Mp * c.d_ff * 2);
    ALLOC_OR_BAIL(h->bh, Mp * d * 4);
    ALLOC_OR_BAIL(h->bq, B * c.n_kv_heads * h->q_rows * c.head_dim * 2);
    h->tm_ok = battn_tc_supported(h->S_max, c.head_dim) &&
               encode_rows_map(&h->tm_q, h->bq, c.head_dim, h->q_rows, (int)(B * c.n_kv_heads)) &&
               encode_rows_map(&h->tm_k, h->kcache, c.head_dim, h->S_max, (int)(c.n_layers * B * c.n_kv_heads)) &&
               encode_rows_map(&h->tm_v, h->vcache, c.head_dim, h->S_max, (int)(c.n_layers * B * c.n_kv_heads));
    if (h->w8a8) {
      ALLOC_OR_BAIL(h->bo8, Mp * c.n_q_heads * c.head_dim);
      ALLOC_OR_BAIL(h->bu8, Mp * c.d_ff);
      ALLOC_OR_BAIL(h->bsa, 4 * Mp * 4);
    }
  }
#undef ALLOC_OR_BAIL
  if (cudaDeviceSynchronize() != cudaSuccess) {
    set_err(h, FM_ERR_CUDA, "set-up failed: %s", cudaGetErrorString(cudaGetLastError()));
    return bail(FM_ERR_CUDA);
  }
  *out = h;
  return FM_OK;
}

namespace {

// Copies the prefix K/V of `batch` requests (k[l], v[l]: [B, p_pad, H_kv, hd],
// request b valid for its first lens[b] rows) into the cache and stores the
// lengths and the chunk's RoPE table on the device.
fm_status set_prefix_impl(fm_expert* h, const uint16_t* const* k, const uint16_t* const* v, int batch,
                          int p_pad, const std::vector<int>& lens, cudaStream_t st) {
  const fm_config& c = h->cfg;
  CK(cudaSetDevice(h->device));
  const size_t per = (size_t)batch * p_pad * c.n_kv_heads * c.head_dim;
  const size_t lay = (size_t)c.max_batch * c.n_kv_heads * h->S_max * c.head_dim;
  void* tmp = nullptr;
  if (p_pad > 0) {
    for (int l = 0; l < c.n_layers; ++l)
      if (!k[l] || !v[l]) return set_err(h, FM_ERR_INVALID_ARG, "prefix pointer of layer %d is NULL", l);
    CK(cudaMalloc(&tmp, per * 2 * 2));
  }
  // lengths first: the copy kernels read them
  CK(cudaMemcpyAsync(h->P_dev, lens.data(), (size_t)batch * 4, cudaMemcpyHostToDevice, st));
  fm_status out = FM_OK;
  for (int l = 0; l < c.n_layers && p_pad > 0; ++l) {
    const uint16_t* srcs[2] = {k[l], v[l]};
    uint16_t* dsts[2] = {h->kcache + l * lay, h->vcache + l * lay};
    for (int i = 0; i < 2; ++i) {
      const uint16_t* src = srcs[i];
      if (!is_device_ptr(src)) {
        uint16_t* t = static_cast<uint16_t*>(tmp) + i * per;
        cudaError_t e = cudaMemcpyAsync(t, src, per * 2, cudaMemcpyDefault, st);
        if (e != cudaSuccess) { out = set_err(h, FM_ERR_CUDA, "prefix upload: %s", cudaGetErrorString(e)); break; }
        src = t;
      }
      cudaError_t e = launch_kv_copy(src, batch, p_pad, h->P_dev, c.n_kv_heads, c.head_dim, h->S_max, dsts[i], st);
      if (e != cudaSuccess) { out = set_err(h, FM_ERR_CUDA, "kv copy: %s", cudaGetErrorString(e)); break; }
    }
    if (out != FM_OK) break;
    if (tmp) {
      // the staging buffer is reused by the next layer
      cudaError_t e = cudaStreamSynchronize(st);
      if (e != cudaSuccess) { out = set_err(h, FM_ERR_CUDA, "prefix sync: %s", cudaGetErrorString(e)); break; }
    }
  }
  if (tmp) cudaFree(tmp);
  if (out != FM_OK) return out;
  CK(launch_rope_table(batch, c.chunk_len, c.head_dim, h->P_dev, (double)c.rope_base, h->rope, st));
  CK(cudaStreamSynchronize(st));
  h->prefix_batch = batch;
  h->prefix_lens = lens;
  return FM_OK;
}

}  // namespace

fm_status fm_set_prefix(fm_expert* h, const uint16_t* const* k, const uint16_t* const* v, int batch,
                        int prefix_len, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, c.max_batch);
  if (prefix_len < 0 || prefix_len > c.max_prefix)
    return set_err(h, FM_ERR_INVALID_ARG, "prefix_len %d outside [0, %d]", prefix_len, c.max_prefix);
  if (prefix_len > 0 && (!k || !v)) return set_err(h, FM_ERR_INVALID_ARG, "k or v is NULL");
  return set_prefix_impl(h, k, v, batch, prefix_len, std::vector<int>(batch, prefix_len),
                         static_cast<cudaStream_t>(stream));
}

fm_status fm_set_prefix_varlen(fm_expert* h, const uint16_t* const* k, const uint16_t* const* v, int batch,
                               const int* prefix_lens, int p_pad, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, c.max_batch);
  if (!prefix_lens) return set_err(h, FM_ERR_INVALID_ARG, "prefix_lens is NULL");
  if (p_pad < 0 || p_pad > c.max_prefix)
    return set_err(h, FM_ERR_INVALID_ARG, "p_pad %d outside [0, %d]", p_pad, c.max_prefix);
  std::vector<int> lens(prefix_lens, prefix_lens + batch);
  for (int b = 0; b < batch; ++b)
    if (lens[b] < 0 || lens[b] > p_pad)
      return set_err(h, FM_ERR_INVALID_ARG, "prefix_lens[%d] = %d outside [0, p_pad = %d]", b, lens[b], p_pad);
  if (p_pad > 0 && (!k || !v)) return set_err(h, FM_ERR_INVALID_ARG, "k or v is NULL");
  return set_prefix_impl(h, k, v, batch, p_pad, lens, static_cast<cudaStream_t>(stream));
}

static fm_status get_graph(fm_expert* h, int batch, int steps, cudaGraphExec_t* out) {
  auto key = std::make_pair(batch, steps);
  auto it = h->graphs.find(key);
  if (it != h->graphs.end()) {
    *out = it->second;
    return FM_OK;
  }
  cudaGraph_t g = nullptr;
  CK(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = enqueue_denoise(h, batch, steps, h->cap_stream);
  cudaError_t e2 = cudaStreamEndCapture(h->cap_stream, &g);
  if (e != cudaSuccess || e2 != cudaSuccess) {
    if (g) cudaGraphDestroy(g);
    return set_err(h, FM_ERR_CUDA, "graph capture: %s / %s", cudaGetErrorString(e), cudaGetErrorString(e2));
  }
  cudaGraphExec_t ex = nullptr;
  e = cudaGraphInstantiate(&ex, g, 0);
  if (e != cudaSuccess) {
    cudaGraphDestroy(g);
    return set_err(h, FM_ERR_CUDA, "graph instantiate: %s", cudaGetErrorString(e));
  }
  h->graphs[key] = ex;
  h->graph_defs[key] = g;
  *out = ex;
  return FM_OK;
}

fm_status fm_denoise(fm_expert* h, const float* x0, int batch, int steps, float* out, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (!x0 || !out) return set_err(h, FM_ERR_INVALID_ARG, "x0 or out is NULL");
  if (steps < 1 || steps > c.max_steps)
    return set_err(h, FM_ERR_INVALID_ARG, "steps %d outside [1, %d]", steps, c.max_steps);
  if (batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, c.max_batch);
  if (h->prefix_batch != batch)
    return set_err(h, FM_ERR_NOT_READY, "fm_set_prefix was not called for batch %d", batch);
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaGraphExec_t ex = nullptr;
  fm_status s = get_graph(h, batch, steps, &ex);
  if (s != FM_OK) return s;
  const size_t bytes = (size_t)batch * c.chunk_len * c.action_dim * 4;
  const bool host_out = !is_device_ptr(out);
  CK(cudaMemcpyAsync(h->x, x0, bytes, cudaMemcpyDefault, st));
  CK(cudaGraphLaunch(ex, st));
  CK(cudaMemcpyAsync(out, h->x, bytes, cudaMemcpyDefault, st));
  if (host_out) {
    CK(cudaStreamSynchronize(st));
    return check_err_word(h);
  }
  return FM_OK;
}

fm_status fm_time_modulation(fm_expert* h, int steps, float* m_out, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (!m_out) return set_err(h, FM_ERR_INVALID_ARG, "m_out is NULL");
  if (steps < 1 || steps > h->cfg.max_steps)
    return set_err(h, FM_ERR_INVALID_ARG, "steps %d outside [1, %d]", steps, h->cfg.max_steps);
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CK(launch_time(time_params(h, steps), h->n_sms, st));
  CK(cudaMemcpyAsync(m_out, h->mod, (size_t)steps * h->n_mod * 4, cudaMemcpyDefault, st));
  CK(cudaStreamSynchronize(st));
  return check_err_word(h);
}

static fm_status velocity_common(fm_expert* h, const float* x, int batch, int step_index, int steps,
                                 cudaStream_t st) {
  const fm_config& c = h->cfg;
  if (!x) return set_err(h, FM_ERR_INVALID_ARG, "x is NULL");
  if (steps < 1 || steps > c.max_steps || step_index < 0 || step_index >= steps)
    return set_err(h, FM_ERR_INVALID_ARG, "step_index %d / steps %d invalid", step_index, steps);
  if (batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, c.max_batch);
  if (h->prefix_batch != batch)
    return set_err(h, FM_ERR_NOT_READY, "fm_set_prefix was not called for batch %d", batch);
  CK(cudaSetDevice(h->device));
  CK(cudaMemcpyAsync(h->x, x, (size_t)batch * c.chunk_len * c.action_dim * 4, cudaMemcpyDefault, st));
  CK(launch_time(time_params(h, steps), h->n_sms, st));
  return FM_OK;
}

fm_status fm_velocity(fm_expert* h, const float* x, int batch, int step_index, int steps, float* v_out,
                      void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (!v_out) return set_err(h, FM_ERR_INVALID_ARG, "v_out is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fm_status s = velocity_common(h, x, batch, step_index, steps, st);
  if (s != FM_OK) return s;
  const fm_config& c = h->cfg;
  const size_t xs = (size_t)c.chunk_len * c.action_dim;
  if (use_batched(h, batch)) {
    CK(enqueue_batched(h, batch, step_index, step_index + 1, steps, false, st));
  } else {
    for (int b = 0; b < batch; ++b) {
      StepParams p = base_params(h);
      p.b = b;
      p.x = h->x + b * xs;
      p.vbuf = h->vbuf + b * xs;
      p.step0 = step_index;
      p.step1 = step_index + 1;
      p.update_x = 0;
      CK(cudaMemsetAsync(h->flags, 0, kFlagBytes, st));
      CK(launch_step(p, st));
    }
  }
  CK(cudaMemcpyAsync(v_out, h->vbuf, (size_t)batch * xs * 4, cudaMemcpyDefault, st));
  if (!is_device_ptr(v_out)) {
    CK(cudaStreamSynchronize(st));
    return check_err_word(h);
  }
  return FM_OK;
}

size_t fm_trace_bytes(const fm_expert* h) {
  if (!h) return 0;
  const fm_config& c = h->cfg;
  const size_t T = c.chunk_len, d = c.d_model, qn = (size_t)c.n_q_heads * c.head_dim,
               kn = (size_t)c.n_kv_heads * c.head_dim;
  const size_t per = T * (d + qn + kn + kn + qn + d + c.d_ff + d);
  return 4 * (c.n_layers * per + T * c.action_dim);
}

namespace {
float bf2f(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}
// Reads element (r, col) of a host copy of an ACT64 matrix.
float act64_get(const std::vector<uint16_t>& a, int r, int col) {
  const size_t idx = (size_t)(col >> 6) * (kRows * 64) + (size_t)r * 64 +
                     ((((col & 63) >> 3) ^ (r & 7)) << 3) + (col & 7);
  return bf2f(a[idx]);
}
float swz_get(const std::vector<uint16_t>& a, size_t row_base, int row, int e) {
  return bf2f(a[row_base + ((((e >> 3) ^ (row & 7))) << 3) + (e & 7)]);
}
}  // namespace

fm_status fm_trace_velocity(fm_expert* h, const float* x, int step_index, int steps, float* trace,
                            void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (!trace) return set_err(h, FM_ERR_INVALID_ARG, "trace is NULL");
  if (h->w8a8) return set_err(h, FM_ERR_UNSUPPORTED, "a W8A8 handle has no one-request kernel to trace");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fm_status s = velocity_common(h, x, 1, step_index, steps, st);
  if (s != FM_OK) return s;
  const fm_config& c = h->cfg;
  const int T = c.chunk_len, d = c.d_model, qn = c.n_q_heads * c.head_dim,
            kn = c.n_kv_heads * c.head_dim, F = c.d_ff, hd = c.head_dim;
  float* out = trace;
  std::vector<float> hbuf((size_t)T * d);
  std::vector<uint16_t> qh((size_t)c.n_kv_heads * h->q_rows * hd), oh((size_t)kRows * qn),
      uh((size_t)kRows * F), kvh((size_t)h->S_max * hd);
  const size_t lay = (size_t)c.max_batch * c.n_kv_heads * h->S_max * hd;
  auto run = [&](int layer0, int layer1, int inproj, int outproj) -> fm_status {
    StepParams p = base_params(h);
    p.step0 = step_index;
    p.step1 = step_index + 1;
    p.layer0 = layer0;
    p.layer1 = layer1;
    p.do_inproj = inproj;
    p.do_outproj = outproj;
    p.update_x = 0;
    p.store_mid = 1;
    CK(cudaMemsetAsync(h->flags, 0, kFlagBytes, st));
    CK(launch_step(p, st));
    CK(cudaStreamSynchronize(st));
    return check_err_word(h);
  };
  // in-proj only (layer range empty)
  if ((s = run(0, 0, 1, 0)) != FM_OK) return s;
  for (int l = 0; l < c.n_layers; ++l) {
    CK(cudaMemcpy(out, h->h_a, (size_t)T * d * 4, cudaMemcpyDeviceToHost));   // h_in
    out += (size_t)T * d;
    if ((s = run(l, l + 1, 0, 0)) != FM_OK) return s;
    CK(cudaMemcpy(qh.data(), h->qbuf, qh.size() * 2, cudaMemcpyDeviceToHost));
    const int G = c.n_q_heads / c.n_kv_heads;
    for (int t = 0; t < T; ++t)
      for (int n = 0; n < qn; ++n) {
        const int head = n / hd, e = n % hd;
        const int row = (head % G) * T + t;
        out[(size_t)t * qn + n] = swz_get(qh, ((size_t)(head / G) * h->q_rows + row) * hd, row, e);
      }
    out += (size_t)T * qn;
    for (int which = 0; which < 2; ++which) {
      const uint16_t* cache = (which == 0 ? h->kcache : h->vcache) + l * lay;
      for (int g = 0; g < c.n_kv_heads; ++g) {
        CK(cudaMemcpy(kvh.data(), cache + (size_t)g * h->S_max * hd, kvh.size() * 2, cudaMemcpyDeviceToHost));
        for (int t = 0; t < T; ++t)
          for (int e = 0; e < hd; ++e) {
            const int row = h->prefix_lens[0] + t;
            out[(size_t)t * kn + g * hd + e] = swz_get(kvh, (size_t)row * hd, row, e);
          }
      }
      out += (size_t)T * kn;
    }
    CK(cudaMemcpy(oh.data(), h->o_act + (size_t)(l & 1) * oh.size(), oh.size() * 2, cudaMemcpyDeviceToHost));
    for (int t = 0; t < T; ++t)
      for (int n = 0; n < qn; ++n) out[(size_t)t * qn + n] = act64_get(oh, t, n);
    out += (size_t)T * qn;
    CK(cudaMemcpy(out, h->h_b, (size_t)T * d * 4, cudaMemcpyDeviceToHost));   // h_mid
    out += (size_t)T * d;
    CK(cudaMemcpy(uh.data(), h->u_act + (size_t)(l & 1) * uh.size(), uh.size() * 2, cudaMemcpyDeviceToHost));
    for (int t = 0; t < T; ++t)
      for (int n = 0; n < F; ++n) out[(size_t)t * F + n] = act64_get(uh, t, n);
    out += (size_t)T * F;
    CK(cudaMemcpy(out, h->h_a, (size_t)T * d * 4, cudaMemcpyDeviceToHost));   // h_out
    out += (size_t)T * d;
  }
  if ((s = run(c.n_layers, c.n_layers, 0, 1)) != FM_OK) return s;
  CK(cudaMemcpy(out, h->vbuf, (size_t)T * c.action_dim * 4, cudaMemcpyDeviceToHost));
  return FM_OK;
}

size_t fm_trace_batched_bytes(const fm_expert* h, int batch) {
  if (!h || batch < 1) return 0;
  const fm_config& c = h->cfg;
  const size_t M = (size_t)batch * c.chunk_len, d = c.d_model, qn = (size_t)c.n_q_heads * c.head_dim,
               kn = (size_t)c.n_kv_heads * c.head_dim;
  return 4 * (c.n_layers * M * (5 * d + 2 * qn + 2 * kn + c.d_ff) + M * c.action_dim);
}

namespace {
// Element (m, k) of a host copy of an ACT128 matrix with K columns.
float act128_get(const std::vector<uint16_t>& a, int K, int m, int k) {
  const size_t blk = ((size_t)(m >> 7) * (K >> 6) + (k >> 6)) * (kBM * 64);
  const int r = m & 127;
  return bf2f(a[blk + (size_t)r * 64 + ((((k & 63) >> 3) ^ (r & 7)) << 3) + (k & 7)]);
}
// Value (code x row scale) of element (m, k) of a host copy of an ACT8 matrix.
float act8_get(const std::vector<uint8_t>& a, const std::vector<float>& sa, int K, int m, int k) {
  const size_t blk = ((size_t)(m >> 7) * (K >> 7) + (k >> 7)) * (kBM * 128);
  const int r = m & 127;
  const uint8_t q = a[blk + (size_t)r * 128 + ((((k & 127) >> 4) ^ (r & 7)) << 4) + (k & 15)];
  // E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; 0x7F / 0xFF are NaN
  const int e = (q >> 3) & 15, mt = q & 7;
  float v = (q & 0x7F) == 0x7F ? NAN : e == 0 ? std::ldexp((float)mt, -9) : std::ldexp(1.0f + mt / 8.0f, e - 7);
  return ((q & 0x80) ? -v : v) * sa[m];
}
}  // namespace

fm_status fm_trace_batched(fm_expert* h, const float* x, int batch, int step_index, int steps, float* trace,
                           void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (!trace) return set_err(h, FM_ERR_INVALID_ARG, "trace is NULL");
  if (!use_batched(h, batch))
    return set_err(h, FM_ERR_UNSUPPORTED, "batch %d does not run on the batched path of this handle", batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  fm_status s = velocity_common(h, x, batch, step_index, steps, st);
  if (s != FM_OK) return s;
  const fm_config& c = h->cfg;
  const int T = c.chunk_len, d = c.d_model, qn = c.n_q_heads * c.head_dim, kn = c.n_kv_heads * c.head_dim,
            F = c.d_ff, hd = c.head_dim, M = batch * T, L = c.n_layers, G = c.n_q_heads / c.n_kv_heads;
  const size_t Mp = (size_t)h->Mp;
  const size_t lay = (size_t)c.max_batch * c.n_kv_heads * h->S_max * hd;
  std::vector<uint16_t> a16;
  std::vector<uint8_t> a8;
  std::vector<float> sa, hbuf((size_t)M * d);
  std::vector<uint16_t> qh((size_t)batch * c.n_kv_heads * h->q_rows * hd), kvh;
  float* out = trace;
  // copies matrix `src` (ACT128 bf16, or ACT8 codes with row scales `scale`
  // on a W8A8 handle) of K columns into out[M][K]
  auto put_act = [&](const void* src, const float* scale, int K) -> cudaError_t {
    cudaError_t e;
    if (scale != nullptr) {
      a8.resize(Mp * K);
      sa.resize(Mp);
      e = cudaMemcpy(a8.data(), src, a8.size(), cudaMemcpyDeviceToHost);
      if (e == cudaSuccess) e = cudaMemcpy(sa.data(), scale, Mp * 4, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return e;
      for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) out[(size_t)m * K + k] = act8_get(a8, sa, K, m, k);
    } else {
      a16.resize(Mp * K);
      e = cudaMemcpy(a16.data(), src, a16.size() * 2, cudaMemcpyDeviceToHost);
      if (e != cudaSuccess) return e;
      for (int m = 0; m < M; ++m)
        for (int k = 0; k < K; ++k) out[(size_t)m * K + k] = act128_get(a16, K, m, k);
    }
    out += (size_t)M * K;
    return cudaSuccess;
  };
  auto put_h = [&]() -> cudaError_t {
    // rows of the residual are d apart, the first M of Mp
    cudaError_t e = cudaMemcpy(out, h->bh, (size_t)M * d * 4, cudaMemcpyDeviceToHost);
    out += (size_t)M * d;
    return e;
  };
  const float* sa_za = h->w8a8 ? h->bsa : nullptr;
  const float* sa_zf = h->w8a8 ? h->bsa + 2 * Mp : nullptr;
  BatchHook hook = [&](int l, int k) -> cudaError_t {
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return e;
    switch (k) {
      case 0:
        e = put_h();
        if (e == cudaSuccess) e = put_act(h->bz_a, sa_za, d);
        return e;
      case 1: {
        e = cudaMemcpy(qh.data(), h->bq, qh.size() * 2, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return e;
        for (int m = 0; m < M; ++m) {
          const int b = m / T, t = m % T;
          for (int n = 0; n < qn; ++n) {
            const int head = n / hd, el = n % hd, row = (head % G) * T + t;
            const size_t base = (((size_t)b * c.n_kv_heads + head / G) * h->q_rows + row) * hd;
            out[(size_t)m * qn + n] = swz_get(qh, base, row, el);
          }
        }
        out += (size_t)M * qn;
        kvh.resize(lay);
        for (int which = 0; which < 2; ++which) {
          e = cudaMemcpy(kvh.data(), (which == 0 ? h->kcache : h->vcache) + l * lay, lay * 2,
                         cudaMemcpyDeviceToHost);
          if (e != cudaSuccess) return e;
          for (int m = 0; m < M; ++m) {
            const int b = m / T, t = m % T, row = h->prefix_lens[b] + t;
            for (int n = 0; n < kn; ++n) {
              const size_t base = (((size_t)b * c.n_kv_heads + n / hd) * h->S_max + row) * hd;
              out[(size_t)m * kn + n] = swz_get(kvh, base, row, n % hd);
            }
          }
          out += (size_t)M * kn;
        }
        return cudaSuccess;
      }
      case 2: return put_act(h->bo, nullptr, qn);
      case 3: return put_h();
      case 4: return put_act(h->bz_f, sa_zf, d);
      case 5: return put_act(h->bu, nullptr, F);
      case 6: return put_h();
      default:
        e = cudaMemcpy(out, h->vbuf, (size_t)M * c.action_dim * 4, cudaMemcpyDeviceToHost);
        out += (size_t)M * c.action_dim;
        return e;
    }
  };
  (void)L;
  (void)hbuf;
  CK(enqueue_batched(h, batch, step_index, step_index + 1, steps, false, st, &hook));
  CK(cudaStreamSynchronize(st));
  return check_err_word(h);
}

fm_status fm_set_prefix_builder(fm_expert* h, const fm_prefix_weights* w, int d_prefix) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (!w) return set_err(h, FM_ERR_INVALID_ARG, "weights are NULL");
  if (d_prefix < 64 || d_prefix % 64 != 0)
    return set_err(h, FM_ERR_INVALID_ARG, "d_prefix %d must be a positive multiple of 64", d_prefix);
  if (h->pre_d != 0) return set_err(h, FM_ERR_INVALID_ARG, "the prefix builder is already loaded");
  const int kn = c.n_kv_heads * c.head_dim, N = 2 * kn;
  if (N % 128 != 0 || (c.head_dim != 64 && c.head_dim != 128))
    return set_err(h, FM_ERR_UNSUPPORTED, "prefix builder needs 2 H_kv hd a multiple of 128, hd 64 or 128");
  CK(cudaSetDevice(h->device));
  const int bn = bgemm_bn(BE_QKV, N), nkb = d_prefix / 64;
  std::vector<PackChunk> jobs;
  std::vector<int32_t> rows;
  for (int nt = 0; nt < N / bn; ++nt) {
    const uint32_t roff = (uint32_t)rows.size();
    for (int q = 0; q < bn; ++q) rows.push_back(nt * bn + q);
    for (int kb = 0; kb < nkb; ++kb) {
      PackChunk pc{};
      pc.dst_off = ((uint64_t)nt * nkb + kb) * bn * 128;
      pc.rowidx_off = roff;
      pc.nrows = (uint16_t)bn;
      pc.mat = 0;
      pc.kb = (uint32_t)kb;
      jobs.push_back(pc);
    }
  }
  h->pre_layer_bytes = (uint64_t)N * d_prefix * 2;
  const size_t Mp = (size_t)((c.max_batch * std::max(c.max_prefix, 1) + kBM - 1) / kBM * kBM);
  DALLOC(h->pre_arena, (size_t)c.n_layers * h->pre_layer_bytes);
  DALLOC(h->pre_stage, Mp * d_prefix * 2);
  DALLOC(h->pre_rows, (size_t)c.max_batch * std::max(c.max_prefix, 1) * d_prefix * 2);
  DALLOC(h->pre_rope, (size_t)std::max(c.max_prefix, 1) * c.head_dim * 4);
  DALLOC(h->pre_zero, 4);   // zero-filled: positions start at 0
  void* tmp = nullptr;
  void* tab = nullptr;
  cudaError_t e = cudaMalloc(&tmp, (size_t)N * d_prefix * 2);
  if (e == cudaSuccess) e = cudaMalloc(&tab, jobs.size() * sizeof(PackChunk) + rows.size() * 4 + 2 * sizeof(void*) + 64);
  fm_status st = FM_OK;
  if (e != cudaSuccess) st = set_err(h, FM_ERR_OOM, "prefix builder staging: %s", cudaGetErrorString(e));
  PackChunk* d_jobs = static_cast<PackChunk*>(tab);
  int32_t* d_rows = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(tab) + jobs.size() * sizeof(PackChunk));
  uint8_t* tail = reinterpret_cast<uint8_t*>(d_rows) + rows.size() * 4;
  tail = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tail) + 15) & ~uintptr_t(15));
  uint16_t** d_mats = reinterpret_cast<uint16_t**>(tail);
  int* d_matk = reinterpret_cast<int*>(tail + sizeof(void*));
  if (st == FM_OK) {
    uint16_t* mp = static_cast<uint16_t*>(tmp);
    e = cudaMemcpy(d_jobs, jobs.data(), jobs.size() * sizeof(PackChunk), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d_rows, rows.data(), rows.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d_mats, &mp, sizeof(void*), cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(d_matk, &d_prefix, sizeof(int), cudaMemcpyHostToDevice);
    for (int l = 0; l < c.n_layers && e == cudaSuccess; ++l) {
      if (!w[l].wk || !w[l].wv) {
        st = set_err(h, FM_ERR_INVALID_ARG, "prefix builder layer %d has a NULL weight", l);
        break;
      }
      e = cudaMemcpy(mp, w[l].wk, (size_t)kn * d_prefix * 2, cudaMemcpyDefault);
      if (e == cudaSuccess) e = cudaMemcpy(mp + (size_t)kn * d_prefix, w[l].wv, (size_t)kn * d_prefix * 2, cudaMemcpyDefault);
      if (e == cudaSuccess)
        e = launch_pack(d_jobs, (int)jobs.size(), d_rows, d_mats, d_matk, h->pre_arena + (size_t)l * h->pre_layer_bytes, 0);
    }
    if (e == cudaSuccess)
      e = launch_rope_table(1, std::max(c.max_prefix, 1), c.head_dim, h->pre_zero, (double)c.rope_base, h->pre_rope, 0);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess && st == FM_OK) st = set_err(h, FM_ERR_CUDA, "prefix builder packing: %s", cudaGetErrorString(e));
  }
  if (tmp) cudaFree(tmp);
  if (tab) cudaFree(tab);
  if (st == FM_OK) h->pre_d = d_prefix;
  return st;
}

fm_status fm_build_prefix(fm_expert* h, const uint16_t* const* hidden, int batch, int prefix_len, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (h->pre_d == 0) return set_err(h, FM_ERR_NOT_READY, "fm_set_prefix_builder was not called");
  if (batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d outside [1, %d]", batch, c.max_batch);
  if (prefix_len < 0 || prefix_len > c.max_prefix)
    return set_err(h, FM_ERR_INVALID_ARG, "prefix_len %d outside [0, %d]", prefix_len, c.max_prefix);
  if (prefix_len > 0 && !hidden) return set_err(h, FM_ERR_INVALID_ARG, "hidden is NULL");
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int d = h->pre_d, kn = c.n_kv_heads * c.head_dim, L = c.n_layers;
  const int M = batch * prefix_len, Mp = (M + kBM - 1) / kBM * kBM;
  const size_t lay = (size_t)c.max_batch * c.n_kv_heads * h->S_max * c.head_dim;
  std::vector<int> lens(batch, prefix_len);
  CK(cudaMemcpyAsync(h->P_dev, lens.data(), (size_t)batch * 4, cudaMemcpyHostToDevice, st));
  BGemmParams g{};
  g.M = M;
  g.Mp = Mp;
  g.K = d;
  g.N = 2 * kn;
  g.T = prefix_len;            // rows m = b * P + p
  g.Hq = 0;                    // no query heads: columns are K heads then V heads
  g.Hkv = c.n_kv_heads;
  g.hd = c.head_dim;
  g.S_max = h->S_max;
  g.rope = h->pre_rope;
  g.rope_stride_b = 0;         // positions 0 .. P-1 for every request
  g.P_dev = nullptr;           // cache rows start at 0
  g.err = h->err_word;
  g.spin_budget = 4000000000LL;
  for (int l = 0; l < L && M > 0; ++l) {
    if (!hidden[l]) return set_err(h, FM_ERR_INVALID_ARG, "hidden states of layer %d are NULL", l);
    const uint16_t* src = hidden[l];
    if (!is_device_ptr(src)) {
      CK(cudaMemcpyAsync(h->pre_rows, src, (size_t)M * d * 2, cudaMemcpyHostToDevice, st));
      src = h->pre_rows;
    }
    CK(launch_rows_to_act128(src, M, Mp, d, h->pre_stage, st));
    g.A = reinterpret_cast<const uint8_t*>(h->pre_stage);
    g.W = h->pre_arena + (size_t)l * h->pre_layer_bytes;
    g.kc = h->kcache + l * lay;
    g.vc = h->vcache + l * lay;
    CK(launch_bgemm(g, BE_QKV, h->n_sms, st));
  }
  CK(launch_rope_table(batch, c.chunk_len, c.head_dim, h->P_dev, (double)c.rope_base, h->rope, st));
  CK(cudaStreamSynchronize(st));
  h->prefix_batch = batch;
  h->prefix_lens = lens;
  return check_err_word(h);
}

fm_status fm_get_prefix_kv(fm_expert* h, int layer, int request, uint16_t* k, uint16_t* v) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (layer < 0 || layer >= c.n_layers || request < 0 || request >= h->prefix_batch || !k || !v)
    return set_err(h, FM_ERR_INVALID_ARG, "layer %d / request %d invalid or NULL buffer", layer, request);
  CK(cudaSetDevice(h->device));
  const int P = h->prefix_lens[request], hd = c.head_dim, Hkv = c.n_kv_heads;
  const size_t lay = (size_t)c.max_batch * Hkv * h->S_max * hd;
  std::vector<uint16_t> buf((size_t)h->S_max * hd);
  for (int which = 0; which < 2; ++which) {
    uint16_t* out = which == 0 ? k : v;
    const uint16_t* cache = (which == 0 ? h->kcache : h->vcache) + layer * lay;
    for (int g = 0; g < Hkv; ++g) {
      CK(cudaMemcpy(buf.data(), cache + (((size_t)request * Hkv + g) * h->S_max) * hd, (size_t)P * hd * 2,
                    cudaMemcpyDeviceToHost));
      for (int p = 0; p < P; ++p)
        for (int e = 0; e < hd; ++e)
          out[((size_t)p * Hkv + g) * hd + e] = buf[(size_t)p * hd + ((((e >> 3) ^ (p & 7))) << 3) + (e & 7)];
    }
  }
  return FM_OK;
}

fm_status fm_get_fp8_weights(fm_expert* h, int layer, int which, uint8_t* codes, float* scale) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (c.wtype == FM_W_BF16) return set_err(h, FM_ERR_INVALID_ARG, "handle holds bf16 weights");
  if (c.wtype == FM_W_FP8_NVFP4_GU && (which == 4 || which == 5))
    return set_err(h, FM_ERR_INVALID_ARG, "gate_up is NVFP4 in this handle (fm_get_nvfp4_weights)");
  if (layer < 0 || layer >= c.n_layers || which < 0 || which > 6 || !codes || !scale)
    return set_err(h, FM_ERR_INVALID_ARG, "layer %d / which %d invalid or NULL buffer", layer, which);
  const int d = c.d_model, F = c.d_ff, qn = c.n_q_heads * c.head_dim, kn = c.n_kv_heads * c.head_dim;
  // linear `which` = rows [r0, r0 + rows) of packed matrix g (K columns)
  static const int kG[7] = {G_QKV, G_QKV, G_QKV, G_O, G_GU, G_GU, G_DOWN};
  const int g = kG[which];
  const int r0s[7] = {0, qn, qn + kn, 0, 0, F, 0};
  const int nrows[7] = {qn, kn, kn, d, F, F, d};
  const int kdim[4] = {d, qn, d, F};
  const int mrows[4] = {qn + 2 * kn, d, 2 * F, d};
  const int r0 = r0s[which], R = nrows[which], K = kdim[g];
  CK(cudaSetDevice(h->device));
  size_t base = (size_t)layer * (mrows[0] + mrows[1] + mrows[2] + mrows[3]);
  for (int i = 0; i < g; ++i) base += mrows[i];
  if (h->w8a8) {
    // tile arena: chunk rows of 128 codes, 16-byte pieces swizzled by (row & 7)
    std::vector<uint8_t> lay(h->blayer_bytes);
    CK(cudaMemcpy(lay.data(), h->barena + (size_t)layer * h->blayer_bytes, h->blayer_bytes, cudaMemcpyDeviceToHost));
    std::memset(codes, 0, (size_t)R * K);
    for (const PackChunk& pc : h->bpack_jobs) {
      if (pc.mat != g) continue;
      for (int q = 0; q < pc.nrows; ++q) {
        const int sr = h->bpack_rows[pc.rowidx_off + q];
        if (sr < r0 || sr >= r0 + R) continue;
        for (int j = 0; j < 8; ++j)
          std::memcpy(codes + (size_t)(sr - r0) * K + (size_t)pc.kb * 128 + j * 16,
                      lay.data() + pc.dst_off + (size_t)q * 128 + ((j ^ (q & 7)) << 4), 16);
      }
    }
    std::memcpy(scale, h->row_scale.data() + base + r0, (size_t)R * 4);
    return FM_OK;
  }
  std::vector<uint8_t> lay(h->layer_bytes);
  CK(cudaMemcpy(lay.data(), h->arena + (size_t)layer * h->layer_bytes, h->layer_bytes, cudaMemcpyDeviceToHost));
  std::memset(codes, 0, (size_t)R * K);
  for (const PackChunk& pc : h->pack_jobs) {
    if (pc.mat != g) continue;
    for (int q = 0; q < pc.nrows; ++q) {
      const int sr = h->pack_rows[pc.rowidx_off + q];
      if (sr < r0 || sr >= r0 + R) continue;
      std::memcpy(codes + (size_t)(sr - r0) * K + (size_t)pc.kb * 64, lay.data() + pc.dst_off + (size_t)q * 64, 64);
    }
  }
  std::memcpy(scale, h->row_scale.data() + base + r0, (size_t)R * 4);
  return FM_OK;
}

fm_status fm_quantize_act_e4m3(fm_expert* h, const uint16_t* x, int M, int K, uint8_t* codes, float* scales,
                               void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (!x || !codes || !scales || M < 1 || K < 256 || K % 256 != 0 || K > 4096)
    return set_err(h, FM_ERR_INVALID_ARG, "M %d / K %d invalid or NULL buffer", M, K);
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Mp = (M + kBM - 1) / kBM * kBM;
  uint16_t* rows = nullptr;
  uint16_t* act = nullptr;
  uint8_t* q = nullptr;
  float* sc = nullptr;
  std::vector<uint8_t> hq((size_t)Mp * K);
  cudaError_t e = cudaMalloc(&rows, (size_t)M * K * 2);
  if (e == cudaSuccess) e = cudaMalloc(&act, (size_t)Mp * K * 2);
  if (e == cudaSuccess) e = cudaMalloc(&q, (size_t)Mp * K);
  if (e == cudaSuccess) e = cudaMalloc(&sc, (size_t)Mp * 4);
  if (e == cudaSuccess) e = cudaMemcpyAsync(rows, x, (size_t)M * K * 2, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = launch_rows_to_act128(rows, M, Mp, K, act, st);
  if (e == cudaSuccess) e = launch_browquant(BQuantParams{act, q, sc, M, K}, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(hq.data(), q, hq.size(), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(scales, sc, (size_t)M * 4, cudaMemcpyDefault, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  for (void* p : {static_cast<void*>(rows), static_cast<void*>(act), static_cast<void*>(q), static_cast<void*>(sc)})
    if (p) cudaFree(p);
  if (e != cudaSuccess) return set_err(h, FM_ERR_CUDA, "quantize: %s", cudaGetErrorString(e));
  // ACT8: blocks of 128 rows x 128 codes, 16-byte pieces swizzled by (m & 7)
  for (int m = 0; m < M; ++m)
    for (int c = 0; c < K; c += 16)
      std::memcpy(codes + (size_t)m * K + c,
                  hq.data() + ((size_t)(m >> 7) * (K >> 7) + (c >> 7)) * (kBM * 128) + (size_t)(m & 127) * 128 +
                      ((((c & 127) >> 4) ^ (m & 7)) << 4),
                  16);
  return FM_OK;
}

fm_status fm_get_nvfp4_weights(fm_expert* h, int layer, int which, uint8_t* codes, uint8_t* block_scales,
                               float* g) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (c.wtype != FM_W_FP8_NVFP4_GU) return set_err(h, FM_ERR_INVALID_ARG, "handle has no NVFP4 weights");
  if (layer < 0 || layer >= c.n_layers || (which != 4 && which != 5) || !codes || !block_scales || !g)
    return set_err(h, FM_ERR_INVALID_ARG, "layer %d / which %d invalid or NULL buffer", layer, which);
  const int d = c.d_model, F = c.d_ff, r0 = which == 4 ? 0 : F;
  CK(cudaSetDevice(h->device));
  std::vector<uint8_t> lay(h->layer_bytes);
  CK(cudaMemcpy(lay.data(), h->arena + (size_t)layer * h->layer_bytes, h->layer_bytes, cudaMemcpyDeviceToHost));
  std::memset(codes, 0, (size_t)F * d);
  std::memset(block_scales, 0, (size_t)F * (d / 16));
  for (const PackChunk& pc : h->pack_jobs) {
    if (pc.mat != G_GU) continue;
    const int R = pc.nrows;
    for (int q = 0; q < R; ++q) {
      const int sr = h->pack_rows[pc.rowidx_off + q];
      if (sr < r0 || sr >= r0 + F) continue;
      const uint8_t* crow = lay.data() + pc.dst_off + (size_t)q * 32;
      const uint8_t* srow = lay.data() + pc.dst_off + (size_t)R * 32 + (size_t)q * 4;
      uint8_t* out = codes + (size_t)(sr - r0) * d + (size_t)pc.kb * 64;
      for (int i = 0; i < 32; ++i) {
        out[2 * i] = crow[i] & 0xF;
        out[2 * i + 1] = crow[i] >> 4;
      }
      std::memcpy(block_scales + (size_t)(sr - r0) * (d / 16) + (size_t)pc.kb * 4, srow, 4);
    }
  }
  *g = h->nv4_g[2 * layer + (which == 4 ? 0 : 1)];
  return FM_OK;
}

fm_status fm_profile_denoise(fm_expert* h, int batch, int steps, int iters, float* ms, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (!ms || iters < 1) return set_err(h, FM_ERR_INVALID_ARG, "ms is NULL or iters < 1");
  if (steps < 1 || steps > c.max_steps || batch < 1 || batch > c.max_batch)
    return set_err(h, FM_ERR_INVALID_ARG, "batch %d / steps %d invalid", batch, steps);
  if (h->prefix_batch != batch)
    return set_err(h, FM_ERR_NOT_READY, "fm_set_prefix was not called for batch %d", batch);
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev[3];
  for (auto& e : ev) CK(cudaEventCreate(&e));
  double t_time = 0.0, t_loop = 0.0;
  const size_t xs = (size_t)c.chunk_len * c.action_dim;
  fm_status out = FM_OK;
  for (int i = 0; i < iters && out == FM_OK; ++i) {
    cudaError_t e = cudaEventRecord(ev[0], st);
    if (e == cudaSuccess) e = launch_time(time_params(h, steps), h->n_sms, st);
    if (e == cudaSuccess) e = cudaEventRecord(ev[1], st);
    if (e == cudaSuccess && use_batched(h, batch)) e = enqueue_batched(h, batch, 0, steps, steps, true, st);
    for (int b = 0; b < batch && e == cudaSuccess && !use_batched(h, batch); ++b) {
      StepParams p = base_params(h);
      p.b = b;
      p.x = h->x + b * xs;
      p.vbuf = h->vbuf + b * xs;
      p.step1 = steps;
      p.dt = -1.0f / (float)steps;
      e = cudaMemsetAsync(h->flags, 0, kFlagBytes, st);
      if (e == cudaSuccess) e = launch_step(p, st);
    }
    if (e == cudaSuccess) e = cudaEventRecord(ev[2], st);
    if (e == cudaSuccess) e = cudaEventSynchronize(ev[2]);
    float a = 0.f, b2 = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&a, ev[0], ev[1]);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&b2, ev[1], ev[2]);
    if (e != cudaSuccess) out = set_err(h, FM_ERR_CUDA, "profile: %s", cudaGetErrorString(e));
    t_time += a;
    t_loop += b2;
  }
  for (auto& e : ev) cudaEventDestroy(e);
  if (out != FM_OK) return out;
  ms[0] = (float)(t_time / iters);
  ms[1] = (float)(t_loop / iters);
  return check_err_word(h);
}

fm_status fm_profile_phases(fm_expert* h, int steps, uint64_t* out, size_t* n, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  const fm_config& c = h->cfg;
  if (!n) return set_err(h, FM_ERR_INVALID_ARG, "n is NULL");
  if (h->w8a8) return set_err(h, FM_ERR_UNSUPPORTED, "a W8A8 handle has no one-request kernel to profile");
  if (steps < 1 || steps > c.max_steps) return set_err(h, FM_ERR_INVALID_ARG, "steps %d invalid", steps);
  const int n_phases = steps * (2 + 5 * c.n_layers), n_gemms = steps * 4 * c.n_layers;
  int per_layer = 0;
  for (int g = 0; g < 4; ++g) per_layer += h->plan[g].nchunk;
  const int n_chunks = steps * c.n_layers * per_layer;
  const int stride = 16 * n_phases + 2 * n_gemms + 2 * n_chunks;
  const size_t need = (size_t)h->n_ctas * stride;
  if (!out) {
    *n = need;
    return FM_OK;
  }
  if (*n < need) return set_err(h, FM_ERR_INVALID_ARG, "out holds %zu values, %zu needed", *n, need);
  if (h->prefix_batch < 1) return set_err(h, FM_ERR_NOT_READY, "fm_set_prefix was not called");
  CK(cudaSetDevice(h->device));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned long long* d = nullptr;
  CK(cudaMalloc(&d, need * 8));
  cudaError_t e = cudaMemsetAsync(d, 0, need * 8, st);
  if (e == cudaSuccess) e = launch_time(time_params(h, steps), h->n_sms, st);
  StepParams p = base_params(h);
  p.step1 = steps;
  p.dt = -1.0f / (float)steps;
  p.tlog = d;
  p.tlog_stride = stride;
  p.tlog_mma_off = 16 * n_phases;
  p.tlog_chunk_off = 16 * n_phases + 2 * n_gemms;
  p.tlog_chunks = n_chunks;
  if (e == cudaSuccess) e = cudaMemsetAsync(h->flags, 0, kFlagBytes, st);
  if (e == cudaSuccess) e = launch_step(p, st);
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, d, need * 8, cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(d);
  if (e != cudaSuccess) return set_err(h, FM_ERR_CUDA, "profile phases: %s", cudaGetErrorString(e));
  *n = need;
  return check_err_word(h);
}

fm_status fm_test_stall(fm_expert* h, int on, long long spin_cycles) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (spin_cycles < 0) return set_err(h, FM_ERR_INVALID_ARG, "spin_cycles %lld is negative", spin_cycles);
  CK(cudaSetDevice(h->device));
  CK(cudaDeviceSynchronize());
  h->test_stall = on ? 1 : 0;
  h->test_spin = spin_cycles;
  // captured graphs hold the old launch parameters
  for (auto& kv : h->graphs) cudaGraphExecDestroy(kv.second);
  for (auto& kv : h->graph_defs) cudaGraphDestroy(kv.second);
  h->graphs.clear();
  h->graph_defs.clear();
  return FM_OK;
}

fm_status fm_sync(fm_expert* h, void* stream) {
  if (!h) return FM_ERR_INVALID_ARG;
  CK(cudaSetDevice(h->device));
  CK(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
  return check_err_word(h);
}

fm_status fm_get_geometry(const fm_expert* h, int* cluster_size, int* n_clusters, int* n_ctas) {
  if (!h) return FM_ERR_INVALID_ARG;
  if (cluster_size) *cluster_size = kClusterSize;
  if (n_clusters) *n_clusters = h->n_clusters;
  if (n_ctas) *n_ctas = h->n_ctas;
  return FM_OK;
}

size_t fm_expert_destroy(fm_expert* h) {
  if (!h) return 0;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  const size_t n = h->bytes;
  free_all(h);
  delete h;
  return n;
}

#pragma GCC visibility pop
}  // extern "C"
