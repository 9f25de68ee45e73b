// fm_time_modulation_noalloc: the time-conditioning MLP for callers that
// must not allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they need the
// modulation rows: real-time control loops whose device memory is fixed and
// audited at start-up (an allocation there can stall the loop or exceed the
// budget), and embedders that hand the library only the buffers they own.  This entry point takes the
// caller's device buffers for the inputs (W1, W2) and the output, and keeps
// its one intermediate -- the bf16 hidden activations SiLU(e W1^T), at most
// 64 steps x 1024 wide -- in a file-scope device array instead of memory it
// would allocate.
//
// It computes what fm_time_modulation computes (same sinusoid, fp32 first
// linear, SiLU, hidden activations rounded to bf16, fp32 second linear), but
// with plain CUDA-core dot products over the caller's row-major W1 and W2
// instead of the handle's packed tensor-core layout.  The sums run in another
// order, so results agree to fp32 rounding (a hidden value that lands on a
// bf16 rounding boundary may round the other way).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/fm_expert.h"
#include "fm_launch.h"

namespace {

constexpr int kNaMaxSteps = 64;
constexpr int kNaMaxD = 1024;
constexpr int kNaTimeDim = 256;

// Shared by every call on a device and kept until the process exits: the bf16
// hidden activations [kNaMaxSteps][kNaMaxD] (128 KB).  Calls that overlap on
// the GPU (for example on two streams) race on it.
static __device__ __align__(256) unsigned short g_noalloc_h1[kNaMaxSteps * kNaMaxD];

constexpr int kNaMaxDevices = 64;
std::mutex g_na_mu;
void* g_na_ptr[kNaMaxDevices] = {};
unsigned long long g_na_ctx[kNaMaxDevices] = {};   // context id the address belongs to

// Hidden activations: one block per step; fp64 sinusoid, fp32 sums.  Neither
// kernel of this file uses a local-memory stack (ptxas: 0 bytes), so a launch
// never needs the driver to enlarge the context's local memory.
__global__ void noalloc_embed_kernel(const unsigned short* __restrict__ w1, int d, int steps,
                                     unsigned short* __restrict__ h1) {
  __shared__ float e[kNaTimeDim];
  const int k = blockIdx.x;
  const double t = 1.0 - (double)k / (double)steps;
  const int half = kNaTimeDim / 2;
  for (int j = threadIdx.x; j < half; j += blockDim.x) {
    const double period = 4e-3 * pow(4.0 / 4e-3, (double)j / (double)(half - 1));
    // sin / cos of 2 pi t / period, with the factor pi applied inside the
    // argument reduction (sincospi: no stack frame)
    double sv, cv;
    sincospi(2.0 * t / period, &sv, &cv);
    e[j] = (float)sv;
    e[j + half] = (float)cv;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const unsigned short* w = w1 + (size_t)i * kNaTimeDim;
    float acc = 0.f;
    for (int j = 0; j < kNaTimeDim; j += 2) {
      const unsigned int pair = *reinterpret_cast<const unsigned int*>(w + j);
      acc = fmaf(e[j], __uint_as_float(pair << 16), acc);
      acc = fmaf(e[j + 1], __uint_as_float(pair & 0xFFFF0000u), acc);
    }
    const float h = acc / (1.0f + expf(-acc));
    // round to nearest even bf16
    unsigned int u = __float_as_uint(h);
    u += 0x7FFFu + ((u >> 16) & 1u);
    h1[(size_t)k * kNaMaxD + i] = (unsigned short)(u >> 16);
  }
}

// m[k][j] = sum_i h1[k][i] W2[j][i]: one warp per output row j, the steps'
// hidden rows (bf16) in shared memory.  Steps go in blocks of kNaStepBlock
// with the block's accumulators in registers (compile-time indices, no
// local-memory stack); the weight row is read once per block.
constexpr int kNaStepBlock = 16;
__global__ void noalloc_mod_kernel(const unsigned short* __restrict__ w2, const unsigned short* __restrict__ h1,
                                   int d, int steps, int n_mod, float* __restrict__ m) {
  extern __shared__ unsigned short hs[];   // [steps][d]
  for (int i = threadIdx.x; i < steps * d; i += blockDim.x) hs[i] = h1[(size_t)(i / d) * kNaMaxD + i % d];
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int j = blockIdx.x * warps + (threadIdx.x >> 5); j < n_mod; j += gridDim.x * warps) {
    const unsigned short* w = w2 + (size_t)j * d;
    for (int k0 = 0; k0 < steps; k0 += kNaStepBlock) {
      float acc[kNaStepBlock];
#pragma unroll
      for (int kk = 0; kk < kNaStepBlock; ++kk) acc[kk] = 0.f;
      for (int c = lane * 2; c < d; c += 64) {
        const unsigned int pair = *reinterpret_cast<const unsigned int*>(w + c);
        const float w0 = __uint_as_float(pair << 16), w1v = __uint_as_float(pair & 0xFFFF0000u);
#pragma unroll
        for (int kk = 0; kk < kNaStepBlock; ++kk) {
          if (k0 + kk < steps) {
            const unsigned int hp = *reinterpret_cast<const unsigned int*>(hs + (k0 + kk) * d + c);
            acc[kk] = fmaf(__uint_as_float(hp << 16), w0, fmaf(__uint_as_float(hp & 0xFFFF0000u), w1v, acc[kk]));
          }
        }
      }
#pragma unroll
      for (int kk = 0; kk < kNaStepBlock; ++kk) {
        float v = acc[kk];
        for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0 && k0 + kk < steps) m[(size_t)(k0 + kk) * n_mod + j] = v;
      }
    }
  }
}

// Id of the current device context (0 if it cannot be read).  A context
// destroyed by cudaDeviceReset and created again gets a new id, and the
// array's address has to be looked up again in it.
unsigned long long current_context_id() {
  typedef int (*GetCurrent)(void**);
  typedef int (*GetId)(void*, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
    cudaGetLastError();
    looked_up = true;
  }
  void* ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != 0 || ctx == nullptr ||
      get_id(ctx, &id) != 0)
    return 0;
  return id;
}

// Device address of the scratch array on the current device.  Set-up runs on
// the first call on a device (and again on the first call after that device's
// context was reset): it asks the runtime for the array's address with the
// device current, so make that call before any stream capture.  Host code must
// not hand g_noalloc_h1 itself to a kernel: in host code that name is a
// host-side stand-in, not a device address.  Nothing in the array has to start
// at zero: each call writes every entry it reads before reading it.
fm_status scratch_on_current_device(void** out, const char** why) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNaMaxDevices) {
    cudaGetLastError();
    *why = "no usable current CUDA device";
    return FM_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_na_mu);
  const unsigned long long ctx = current_context_id();
  if (g_na_ptr[dev] == nullptr || ctx == 0 || ctx != g_na_ctx[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_h1);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      *why = "cudaGetSymbolAddress of the scratch array failed";
      return FM_ERR_CUDA;
    }
    g_na_ptr[dev] = p;
    // the look-up made the device's context current if no call had yet
    g_na_ctx[dev] = ctx != 0 ? ctx : current_context_id();
  }
  *out = g_na_ptr[dev];
  return FM_OK;
}

}  // namespace

extern "C" {
#pragma GCC visibility push(default)

fm_status fm_time_modulation_noalloc(const uint16_t* w1, const uint16_t* w2, int d_model, int n_mod,
                                     int steps, float* m_out, void* stream) {
  fm::set_thread_error("");
  if (w1 == nullptr || w2 == nullptr || m_out == nullptr) {
    fm::set_thread_error("fm_time_modulation_noalloc: w1, w2 and m_out must be device pointers, not NULL");
    return FM_ERR_INVALID_ARG;
  }
  if ((reinterpret_cast<uintptr_t>(w1) | reinterpret_cast<uintptr_t>(w2) | reinterpret_cast<uintptr_t>(m_out)) & 3u) {
    fm::set_thread_error("fm_time_modulation_noalloc: w1, w2 and m_out must be 4-byte aligned");
    return FM_ERR_INVALID_ARG;
  }
  if (steps < 1 || steps > kNaMaxSteps || d_model < 64 || d_model > kNaMaxD || d_model % 64 != 0 || n_mod < 1) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "fm_time_modulation_noalloc: steps %d / d_model %d / n_mod %d out of range (1 <= steps <= %d, "
             "64 <= d_model <= %d and a multiple of 64, n_mod >= 1)",
             steps, d_model, n_mod, kNaMaxSteps, kNaMaxD);
    fm::set_thread_error(msg);
    return FM_ERR_INVALID_ARG;
  }
  void* scratch = nullptr;
  const char* why = "";
  const fm_status st = scratch_on_current_device(&scratch, &why);
  if (st != FM_OK) {
    fm::set_thread_error(why);
    return st;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned short* h1 = static_cast<unsigned short*>(scratch);
  noalloc_embed_kernel<<<steps, 256, 0, s>>>(w1, d_model, steps, h1);
  const size_t smem = (size_t)steps * d_model * sizeof(unsigned short);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(noalloc_mod_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
          cudaSuccess) {
    cudaGetLastError();
    fm::set_thread_error("fm_time_modulation_noalloc: shared memory attribute refused");
    return FM_ERR_CUDA;
  }
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  noalloc_mod_kernel<<<sms * 2, 256, smem, s>>>(w2, h1, d_model, steps, n_mod, m_out);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    fm::set_thread_error("fm_time_modulation_noalloc: kernel launch failed");
    return FM_ERR_CUDA;
  }
  return FM_OK;
}

#pragma GCC visibility pop
}  // extern "C"
