// Internal structures shared by the host engine (fm_api.cu) and the kernels.
//
// Data layouts (device memory):
//  * "ACT64": a bf16 activation matrix of 64 rows (rows >= valid tokens are
//    padding) and K columns, stored as K/64 blocks of 8 KB.  Block kb holds
//    columns [64 kb, 64 kb + 64) as 64 rows of 128 bytes; the 16-byte piece c
//    of row r sits at piece (c ^ (r & 7)).  This is the 128-byte-swizzled,
//    K-major image the tensor cores read, so one bulk copy moves a block from
//    global to shared memory ready for tcgen05.mma.
//  * Packed weights: the same image with rows = output channels: a "chunk" is
//    R rows x 64 input columns (R * 128 bytes).  The engine lays every CTA's
//    chunks of one layer out contiguously, in the order the CTA consumes them.
//    With E4M3 weights a chunk is R rows x 64 one-byte codes, plain row-major
//    (R * 64 bytes); the kernel widens it to the bf16 image in shared memory.
//    The per-output-row scales of a layer sit in a table indexed by packed
//    channel (see StepParams::wscale).
//  * KV cache: [L][B][H_kv][S_max][hd] bf16, each 256-byte row (hd = 128)
//    split in 16-byte pieces stored at piece (c ^ (row & 7)); rows 0..P-1 are
//    the prefix, rows P..P+T-1 the chunk of the current velocity evaluation.
//  * q buffer: per KV group g, rows (h % G) * T + t for the G query heads
//    of the group, [H_kv][q_rows][hd] bf16, same per-row piece swizzle.
#pragma once
#include <cstdint>

namespace fm {

constexpr int kClusterSize = 8;        // CTAs per cluster (portable maximum)
constexpr int kMaxClusters = 24;       // 8-CTA clusters a B200 can hold (148 SMs)
constexpr int kComputeWarps = 4;       // warps 2..5
constexpr int kThreads = 192;          // producer warp, MMA warp, 4 compute warps
constexpr int kConvWarps = 2;          // E4M3 -> bf16 widening warps of the step kernel
constexpr int kStepThreads = kThreads + 32 * kConvWarps;
constexpr int kRows = 64;              // MMA M: token rows per tile
constexpr int kMaxT = 50;              // valid token rows (one chunk)
constexpr int kBiasRow = 50;           // row carrying the AdaRMSNorm shift vector
constexpr int kRecvRows = 51;          // rows 0..50 travel in the split-K reduction
constexpr int kTimeDim = 256;
constexpr int kRingSlots = 16;         // mbarrier pairs of the weight ring
constexpr int kRingBytes = 126 * 1024; // weight ring
constexpr int kWorkBytes = 96 * 1024;  // activation / receive region
constexpr int kSmemMax = 232448;       // dynamic shared memory per CTA (227 KB)

enum GemmId { G_QKV = 0, G_O = 1, G_GU = 2, G_DOWN = 3 };

// Hand-offs of the one-request loop kernel.  Each phase's writers add 1 to
// the phase's counter (release) once their outputs are stored; a consumer
// waits (acquire) until the counter reaches rounds x writers.
//   F_Z   z_a, h_a and the h^2 row sums: in-projection / down owners
//   F_ZF  z_f, h_b and the h^2 row sums: o_proj owners
//   F_QKV q buffer and the chunk's K/V cache rows: QKV owners
//   F_O   attention output: attention CTAs
//   F_U   SwiGLU output: gate_up owners
//   F_X   chunk x after the Euler update: every CTA
enum FlagId { F_Z = 0, F_ZF = 1, F_QKV = 2, F_O = 3, F_U = 4, F_X = 5, kNumFlags = 6 };
constexpr int kFlagStride = 32;   // 32-bit words between counters (one 128-byte line each)
constexpr size_t kFlagBytes = (size_t)kNumFlags * kFlagStride * 4;

// One linear of a layer, partitioned over clusters.  Cluster c works on
// NS n-groups of ng[c] packed output channels each (0 = idle cluster); CTA j
// of the cluster takes n-group j / KS and K-slice j % KS (kslice columns).
// After the in-cluster split-K reduction CTA j owns ng[c] / KS consecutive
// columns of its n-group.  Packed channels of cluster c start at ch_off[c]
// (for gate_up: u columns, each n-group holding gate and up rows in pairs).
struct GemmPlan {
  int N;          // logical output channels (gate_up: 2 F packed rows)
  int K;          // reduction length
  int NS, KS;     // n-groups and K-slices per cluster (NS * KS = 8)
  int kslice;     // K per slice (multiple of 64)
  int nchunk;     // kslice / 64: weight chunks and activation blocks per CTA
  int busy_clusters;
  int max_ng;
  int ch_off[kMaxClusters];
  int ng[kMaxClusters];
};

struct StepParams {
  int L, d, Hq, Hkv, hd, F, A, T, S_max;
  int B_cap;                 // request slots in the KV cache
  int b;                     // request handled by this launch
  const int* P_dev;          // [B_cap] prefix length per request, read on the device (no recapture on change)
  float eps;
  int n_clusters, n_ctas;
  GemmPlan g[4];
  // attention: per KV group, G*T query rows (head-major) in blocks of 64
  int att_blocks;            // 64-row blocks per KV group
  int q_rows;                // padded rows per KV group in the q buffer (multiple of 64)
  // weights
  const uint8_t* arena;      // packed per-layer weights (bf16 image or E4M3 codes)
  uint64_t layer_bytes;      // bytes of one layer in the arena
  int wfmt[4];               // per linear: 0 bf16 image, 1 E4M3 rows (64 B), 2 NVFP4 rows
                             // (32 B of codes, then 4 B of block scales per row); 1 and 2
                             // are widened to bf16 in shared memory
  const float* wscale;       // quantised weights: [L][sc_stride] fp32 column scales by packed
                             // channel (E4M3 row scale or NVFP4 tensor scale); bf16: null
  int sc_stride;             // floats per layer in wscale
  int sc_off[4];             // first entry of each linear inside a layer's table
  const uint32_t* span_off;  // [n_ctas + 1]: byte offset of each CTA's span in a layer
  const uint16_t* w_in;      // [d, A] bf16
  const uint16_t* w_out;     // [A, d] bf16
  const float* out_bias;     // [A] or null
  // per-call tables
  const float* mod;          // [steps][n_mod] fp32 modulation rows
  int n_mod;
  const float* rope;         // [B_cap][T][hd/2][2] cos, sin for positions P_b .. P_b+T-1
  // buffers
  float* x;                  // [T, A]
  float* vbuf;               // [T, A]
  float* h_a;                // [T, d]
  float* h_b;                // [T, d]
  // activations of layer l live in copy (l & 1) of each buffer
  uint16_t* z_a;             // 2 x ACT64 [64, d]: h (1 + s_a), row 50 = b_a
  uint16_t* z_f;             // 2 x ACT64 [64, d]: h (1 + s_f), row 50 = b_f
  uint16_t* o_act;           // 2 x ACT64 [64, H_q hd]
  uint16_t* u_act;           // 2 x ACT64 [64, F]
  float* sumsq_a;            // [n_ctas][64] per-CTA partial row sums of h^2
  float* sumsq_f;
  uint16_t* qbuf;            // [H_kv][q_rows][hd]: row (h % G) * T + t of group h / G
  uint16_t* kcache;          // [L][B][H_kv][S_max][hd]
  uint16_t* vcache;
  uint32_t* flags;           // hand-off counters [kNumFlags][kFlagStride], zeroed before
                             // each launch: writer CTAs add 1 (release) per round
  uint32_t* err;             // error word (non-zero: a bounded wait gave up)
  // schedule of this launch
  int step0, step1;          // modulation rows used
  int layer0, layer1;        // layers run per step
  int do_inproj, do_outproj, update_x;
  int store_mid;             // also store h after the attention residual (h_b; per-layer trace only)
  int h_regs;                // o_proj and down have the same owners: h stays in registers
  float dt;
  long long spin_budget;     // cycles before a wait gives up
  int stall_test;            // test hook: one writer too many at the QKV hand-off (that wait
                             // cannot complete; exercises the bounded waits and the abort path)
  // optional phase timeline (globaltimer ns); null when not profiling
  unsigned long long* tlog;  // [n_ctas][tlog_stride]: 8 marks per phase, 2 per GEMM (MMA warp),
  int tlog_stride;           // then per weight chunk: landed (MMA warp) and issued (producer)
  int tlog_mma_off;          // offset of the MMA-warp marks inside a CTA's row
  int tlog_chunk_off;        // offset of the per-chunk marks
  int tlog_chunks;           // chunk slots per section
};

struct TimeParams {
  int n_steps, d, n_mod;
  const uint16_t* w1;        // [d, 256] bf16
  const uint8_t* w2_packed;  // chunks of 128 rows x 64 cols, [n_mod/128][d/64]
  uint16_t* h1_act;          // ACT64 [64, d]
  float* mod;                // [n_steps][n_mod]
  uint32_t* err;
  long long spin_budget;
};

// One packing job: copy `nrows` source rows (row indices from `rowidx`, -1 =
// zero row) x 64 columns starting at column 64*kb into the swizzled image at
// byte offset dst_off.
struct PackChunk {
  uint64_t dst_off;
  uint32_t rowidx_off;
  uint16_t nrows;
  uint8_t mat;
  uint8_t fmt;               // weight format: 0 bf16, 1 E4M3, 2 NVFP4
  uint32_t kb;
};

}  // namespace fm
