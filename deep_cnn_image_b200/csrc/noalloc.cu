// noalloc.cu -- an entry point that needs no caller scratch and allocates
// nothing: the weight gradient of a stride-1 convolution
// (alexnet_op_conv_wgrad_noalloc), with its split-K partial sums kept in a
// fixed-size array that lives in this library's own device memory.
//
// Some callers cannot hand this library scratch memory and cannot let it
// allocate any: code that runs after a framework has reserved the whole
// device through its own allocator, or a service that forbids device
// allocation once it has started.  They pass only inputs and outputs.
//
// The array (kNoAllocScratchBytes) is a file-scope __device__ variable: every
// GPU that loads the library holds it until the process exits.  Host code may
// not pass the variable's name to a kernel (on the host that name is only a
// stand-in, not a device address), so the device address is looked up with
// cudaGetSymbolAddress once per device, with that device current, the first
// time the entry point runs on it.  That first call should therefore come
// before any stream capture.  The cached address belongs to the device's
// context at that time: after cudaDeviceReset (or any other teardown of the
// primary context) it is stale, so the cache is keyed by the context and
// looked up again when the context changes.  All calls share the one array:
// two calls whose work overlaps on the GPU (different streams, or different
// host threads) race on it and must be ordered by the caller.
//
// The array's first 256 bytes hold the status word of the pipelined GEMM's
// bounded waits.  The call clears it, launches, and reads it back before it
// returns, so a wait that ran out is reported as ALEXNET_ERR_TIMEOUT instead
// of a silently wrong gradient; the call therefore returns only once its
// result is in dw.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "alexnet.h"
#include "alexnet_ops.h"
#include "conv_desc.h"
#include "gemm.h"
#include "kernels.h"

using namespace alx;

namespace {

constexpr size_t kNoAllocScratchBytes = 16u << 20;  // 16 MiB
constexpr size_t kStatusBytes = 256;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};

// The calling thread's current context (null if none yet), through the
// driver entry point the runtime hands out (the library links no libcuda).
CUcontext current_ctx() {
  static PFN_cuCtxGetCurrent_v4000 fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      f = nullptr;
    return reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(f);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array on the current device (set-up on the
// first call per device, and again whenever the device's context is a
// different one than at the last look-up).
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  const CUcontext ctx = current_ctx();
  if (!g_noalloc_ptr[dev] || !ctx || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    // (initialises the device's primary context if nothing has yet)
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = current_ctx();
  }
  return g_noalloc_ptr[dev];
}

int noalloc_num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// dw[o, kh, kw, ci] = sum over split s of part[s][g][o - g*Og][(kh*K + kw)*P + ci]
// (P = channels per tap in the partial sums), summed in the order s = 0, 1, ...
__global__ void k_wgrad_sum(const float* __restrict__ part, int S, int Cout, int K, int Cg,
                            int P, int groups, float* __restrict__ dw) {
  const uint32_t n = static_cast<uint32_t>(Cout) * K * K * Cg;
  const int Og = Cout / groups;
  const uint32_t Kc = static_cast<uint32_t>(K) * K * Cg;  // canonical row length
  const uint32_t Kp = static_cast<uint32_t>(K) * K * P;   // partial row length
  const size_t split_stride = static_cast<size_t>(groups) * Og * Kp;
  for (uint32_t p = blockIdx.x * blockDim.x + threadIdx.x; p < n; p += gridDim.x * blockDim.x) {
    const uint32_t inner = p % Kc;
    const uint32_t tap = inner / Cg, ci = inner - tap * Cg;
    const int o = static_cast<int>(p / Kc);
    const int g = o / Og;
    const size_t base = (static_cast<size_t>(g) * Og + (o - g * Og)) * Kp + tap * P + ci;
    float acc = 0.f;
    for (int s = 0; s < S; ++s) acc += part[s * split_stride + base];
    dw[p] = acc;
  }
}

}  // namespace

extern "C" alexnet_status alexnet_op_conv_wgrad_noalloc(const void* x, int B, int H, int W,
                                                        int Cin, const void* dy, int Cout, int K,
                                                        int pad, int groups, int splits,
                                                        float* dw, void* stream) {
  if (!x || !dy || !dw || B < 1 || H < 1 || W < 1 || Cin < 1 || Cout < 1 || K < 1 || pad < 0 ||
      groups < 1 || Cin % groups || Cout % groups)
    return ALEXNET_ERR_INVALID_ARG;
  const ConvShape cs{B, H, W, Cin, Cin / groups, Cout / groups, groups, K, pad};
  if (cs.Cg % 8 || cs.Og % 8 || cs.Ho() < 1 || cs.Wo() < 1) return ALEXNET_ERR_INVALID_ARG;
  const size_t per_split = static_cast<size_t>(Cout) * cs.Kdim() * sizeof(float);
  const size_t room = kNoAllocScratchBytes - kStatusBytes;
  if (per_split > room) return ALEXNET_ERR_UNSUPPORTED;  // one split exceeds the array
  char* scratch = static_cast<char*>(noalloc_scratch());
  if (!scratch) return ALEXNET_ERR_CUDA;
  int* status = reinterpret_cast<int*>(scratch);
  float* part = reinterpret_cast<float*>(scratch + kStatusBytes);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // as many K-slices as asked for (or as fill the GPU), but no more than the
  // array holds
  GemmDesc d;
  if (!conv_desc_wgrad(&d, cs, x, dy, part, splits, noalloc_num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  const int s_fit = static_cast<int>(room / per_split);
  if (d.args.splits > s_fit) {
    if (!conv_desc_wgrad(&d, cs, x, dy, part, s_fit, noalloc_num_sms(), status))
      return ALEXNET_ERR_UNSUPPORTED;
  }
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return ALEXNET_ERR_CUDA;
  if (gemm_launch(d, s) != cudaSuccess) return ALEXNET_ERR_CUDA;
  const uint32_t n = static_cast<uint32_t>(Cout) * K * K * cs.Cg;
  const int grid = static_cast<int>((n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16);
  k_wgrad_sum<<<grid, 256, 0, s>>>(part, d.args.splits, Cout, K, cs.Cg, cs.P(), groups, dw);
  count_launch();
  if (cudaGetLastError() != cudaSuccess) return ALEXNET_ERR_CUDA;
  // the GEMM's status word: a bounded wait that ran out leaves dw invalid
  int st = 0;
  if (cudaMemcpyAsync(&st, status, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return ALEXNET_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return ALEXNET_ERR_CUDA;
  if (st & STATUS_TIMEOUT) return ALEXNET_ERR_TIMEOUT;
  return ALEXNET_OK;
}
