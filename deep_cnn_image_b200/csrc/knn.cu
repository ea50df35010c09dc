// knn.cu -- Euclidean nearest neighbours of feature vectors.
//
// [S] "ImageNet Classification with Deep Convolutional Neural Networks",
// "Qualitative Evaluation" (Figure 4, right): images are retrieved by the
// Euclidean distance between their 4096-dimensional last-hidden-layer
// activations.  For Q query rows q and N base rows x (D features each):
//   d(i, j) = ||q_i||^2 + ||x_j||^2 - 2 q_i . x_j
// The dot products are one tcgen05 GEMM (queries as A, base as B, fp32
// out); the squared norms come from a row kernel; a selection kernel keeps
// each query's k smallest distances (ties to the lower base index).
#include <cuda_bf16.h>

#include <cfloat>
#include <cstdint>
#include <cstring>

#include "alexnet.h"
#include "gemm.h"
#include "kernels.h"

namespace alx {
namespace {

constexpr int kKnnMaxK = 32;

// Squared norm of each bf16 row (one warp per row, 16-byte loads, fp32
// sums; D % 8 == 0 and rows 16-byte aligned).
__global__ void k_row_sqnorm(const __nv_bfloat16* __restrict__ x, int rows, int D,
                             float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const long long warps = 1LL * gridDim.x * (blockDim.x >> 5);
  const int d8 = D >> 3;
  for (long long r = blockIdx.x * 1LL * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps) {
    const uint4* row = reinterpret_cast<const uint4*>(x + r * D);
    float s = 0.f;
    for (int i = lane; i < d8; i += 32) {
      const uint4 u = row[i];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float lo = __uint_as_float(w[t] << 16), hi = __uint_as_float(w[t] & 0xFFFF0000u);
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
      }
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) out[r] = s;
  }
}

// (a, ia) ranks before (b, ib): smaller distance, then lower index.
__device__ __forceinline__ bool before(float a, int ia, float b, int ib) {
  return a < b || (a == b && ia < ib);
}

// One block per query: every thread keeps its k best candidates of a
// strided share of the base (a sorted list, insertion from the tail), then k
// rounds of a block-wide minimum over the threads' list heads pick the
// result in order.  Lists live in registers (all indices compile-time);
// KMAX >= k is their capacity, THREADS the block size (fewer threads for the
// longest lists, which need the most registers).
template <int KMAX, int THREADS>
__global__ void __launch_bounds__(THREADS) k_knn_select(const float* __restrict__ dots, int N,
                                                    const float* __restrict__ qn,
                                                    const float* __restrict__ xn, int k,
                                                    float* __restrict__ dist,
                                                    int32_t* __restrict__ idx) {
  __shared__ float wv[32];
  __shared__ int wi[32], wt[32];
  __shared__ int winner;
  const int q = blockIdx.x;
  const float nq = qn[q];
  float bd[KMAX];
  int bi[KMAX];
#pragma unroll
  for (int t = 0; t < KMAX; ++t) {
    bd[t] = FLT_MAX;
    bi[t] = 0x7fffffff;
  }
  // four consecutive candidates per step (N % 4 == 0, rows 16-byte aligned)
  const float4* row4 = reinterpret_cast<const float4*>(dots + static_cast<size_t>(q) * N);
  const float4* xn4 = reinterpret_cast<const float4*>(xn);
  for (int j4 = threadIdx.x; j4 < (N >> 2); j4 += blockDim.x) {
    const float4 g4 = row4[j4], n4 = xn4[j4];
  #pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float gv = e == 0 ? g4.x : e == 1 ? g4.y : e == 2 ? g4.z : g4.w;
      const float nv = e == 0 ? n4.x : e == 1 ? n4.y : e == 2 ? n4.z : n4.w;
      const int j = 4 * j4 + e;
      const float d = fmaxf(nq + nv - 2.f * gv, 0.f);
      float last = FLT_MAX;
      int last_i = 0x7fffffff;
  #pragma unroll
      for (int t = 0; t < KMAX; ++t)
        if (t == k - 1) {
          last = bd[t];
          last_i = bi[t];
        }
      if (!before(d, j, last, last_i)) continue;
      bool placed = false;
  #pragma unroll
      for (int t = KMAX - 1; t >= 0; --t) {
        if (t < k && !placed) {
          if (t > 0 && before(d, j, bd[t - 1 > 0 ? t - 1 : 0], bi[t - 1 > 0 ? t - 1 : 0])) {
            bd[t] = bd[t - 1 > 0 ? t - 1 : 0];
            bi[t] = bi[t - 1 > 0 ? t - 1 : 0];
          } else {
            bd[t] = d;
            bi[t] = j;
            placed = true;
          }
        }
      }
    }
  }
  int head = 0;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int r = 0; r < k; ++r) {
    float v = FLT_MAX;
    int vi = 0x7fffffff;
#pragma unroll
    for (int t = 0; t < KMAX; ++t)
      if (t == head) {
        v = bd[t];
        vi = bi[t];
      }
    int owner = threadIdx.x;
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, v, o);
      const int oi = __shfl_xor_sync(0xffffffffu, vi, o);
      const int ot = __shfl_xor_sync(0xffffffffu, owner, o);
      if (before(ov, oi, v, vi)) {
        v = ov;
        vi = oi;
        owner = ot;
      }
    }
    if (lane == 0) {
      wv[w] = v;
      wi[w] = vi;
      wt[w] = owner;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float b = wv[0];
      int bix = wi[0], bt = wt[0];
      for (int u = 1; u < static_cast<int>(blockDim.x >> 5); ++u)
        if (before(wv[u], wi[u], b, bix)) {
          b = wv[u];
          bix = wi[u];
          bt = wt[u];
        }
      dist[static_cast<size_t>(q) * k + r] = b;
      idx[static_cast<size_t>(q) * k + r] = bix;
      winner = bt;
    }
    __syncthreads();
    if (threadIdx.x == winner) ++head;
    __syncthreads();
  }
}

int knn_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n < 1) n = 148;
  }
  return n;
}

}  // namespace
}  // namespace alx

using namespace alx;

extern "C" {

size_t alexnet_knn_workspace_bytes(int Q, int N) {
  if (Q < 1 || N < 1) return 0;
  const size_t a = (static_cast<size_t>(Q) * N * sizeof(float) + 255) & ~static_cast<size_t>(255);
  const size_t b = (static_cast<size_t>(Q) * sizeof(float) + 255) & ~static_cast<size_t>(255);
  const size_t c = (static_cast<size_t>(N) * sizeof(float) + 255) & ~static_cast<size_t>(255);
  return a + b + c + 256 + 256;  // + the GEMM's status word, + alignment
}

alexnet_status alexnet_knn_sqnorms(const void* x, int rows, int D, float* out, void* stream) {
  if (!x || !out || rows < 1 || D < 8 || D % 8 || (reinterpret_cast<uintptr_t>(x) & 15))
    return ALEXNET_ERR_INVALID_ARG;
  const long long nb = (static_cast<long long>(rows) + 7) / 8;
  k_row_sqnorm<<<static_cast<unsigned>(nb < 148 * 32 ? nb : 148 * 32), 256, 0,
                 static_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(x), rows,
                                                      D, out);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ALEXNET_OK : ALEXNET_ERR_CUDA;
}

alexnet_status alexnet_knn(const void* queries, int Q, const void* base, int N, int D, int k,
                           const float* base_sqnorm, float* dist, int32_t* idx, void* ws,
                           size_t ws_bytes, void* stream) {
  if (!queries || !base || !dist || !idx || !ws || Q < 1 || N < 1 || D < 8 || k < 1 ||
      k > kKnnMaxK || k > N || N % 8 || D % 8 || ws_bytes < alexnet_knn_workspace_bytes(Q, N) ||
      ((reinterpret_cast<uintptr_t>(queries) | reinterpret_cast<uintptr_t>(base)) & 15))
    return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* p = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(ws) + 255) &
                                    ~static_cast<uintptr_t>(255));
  float* dots = reinterpret_cast<float*>(p);
  p += (static_cast<size_t>(Q) * N * sizeof(float) + 255) & ~static_cast<size_t>(255);
  float* qn = reinterpret_cast<float*>(p);
  p += (static_cast<size_t>(Q) * sizeof(float) + 255) & ~static_cast<size_t>(255);
  float* xn = reinterpret_cast<float*>(p);
  p += (static_cast<size_t>(N) * sizeof(float) + 255) & ~static_cast<size_t>(255);
  int* status = reinterpret_cast<int*>(p);  // a bounded wait that runs out sets a bit here
  // dots[i][j] = q_i . x_j: queries K-major as A, base K-major as B
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_TMA_K;
  d.bsrc = B_TMA_K;
  d.bn = 128;
  GemmArgs& a = d.args;
  a.M = Q;
  a.N = N;
  a.Kblocks = (D + 63) / 64;
  a.kb_per_split = a.Kblocks;
  a.groups = 1;
  a.epi = EPI_F32;
  a.out = dots;
  a.ld_out = N;
  a.split_stride = static_cast<long long>(Q) * N;
  a.status = status;
  const auto* qb = static_cast<const __nv_bfloat16*>(queries);
  const auto* xb = static_cast<const __nv_bfloat16*>(base);
  if (!make_tmap_bf16(&d.tmA, qb, D, Q, static_cast<uint64_t>(D) * 2, 64, 128) ||
      !make_tmap_bf16(&d.tmB, xb, D, N, static_cast<uint64_t>(D) * 2, 64, 128) ||
      !gemm_finalize(&d, knn_sms()))
    return ALEXNET_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return ALEXNET_ERR_CUDA;
  k_row_sqnorm<<<(Q + 7) / 8, 256, 0, s>>>(qb, Q, D, qn);
  count_launch();
  if (base_sqnorm) {
    xn = const_cast<float*>(base_sqnorm);  // read only
  } else {
    const long long nb = (static_cast<long long>(N) + 7) / 8;
    k_row_sqnorm<<<static_cast<unsigned>(nb < 148 * 32 ? nb : 148 * 32), 256, 0, s>>>(xb, N, D,
                                                                                       xn);
    count_launch();
  }
  if (gemm_launch(d, s) != cudaSuccess) return ALEXNET_ERR_CUDA;
  if (k <= 8)
    k_knn_select<8, 512><<<Q, 512, 0, s>>>(dots, N, qn, xn, k, dist, idx);
  else if (k <= 16)
    k_knn_select<16, 512><<<Q, 512, 0, s>>>(dots, N, qn, xn, k, dist, idx);
  else
    k_knn_select<32, 256><<<Q, 256, 0, s>>>(dots, N, qn, xn, k, dist, idx);
  count_launch();
  return cudaGetLastError() == cudaSuccess ? ALEXNET_OK : ALEXNET_ERR_CUDA;
}

}  // extern "C"
