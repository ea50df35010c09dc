// kernels.cu -- the memory-bound kernels of the AlexNet training step.
//
// Pages cited:
//   [S] "ImageNet Classification with Deep Convolutional Neural Networks",
//       paper-graph-ui summary page, section 3.4 subsections.
//   [W] "AlexNet and Deep CNNs" (fermi.ai wiki page).
// Layout: NHWC bf16 activations, channels fastest; each thread moves one
// 16-byte chunk (8 channels) so every load and store is a full vector.
#include <cuda_bf16.h>

#include <atomic>

#include "kernels.h"
#include "ptx.cuh"

namespace alx {

namespace {

constexpr int kMaxGrid = 148 * 16;

inline int grid_for(long long n, int block) {
  long long g = (n + block - 1) / block;
  if (g > kMaxGrid) g = kMaxGrid;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) { unpack8_bits(u, f); }
__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}
__device__ __forceinline__ float2 ld_bf16x2(const bf16* p) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(bf16_lo(u), bf16_hi(u));
}

// LRN powers of the scale s = k + alpha * sum a^2 (s >= k > 0): s^(-beta),
// and s^(-beta-1) for the backward.  For beta = 3/4, the pages' value, both
// come from two reciprocal square roots: q = s^(-1/2), r = q^(-1/2) = s^(1/4),
// s^(-3/4) = q^2 r, s^(-7/4) = s^(-3/4) q^2.  Otherwise s^(-beta) is
// exp2(-beta log2 s) and s^(-beta-1) = s^(-beta) / s.
template <bool B34>
__device__ __forceinline__ float lrn_pow(float sc, float beta) {
  if (B34) {
    const float q = rsqrt_approx(sc);
    return q * q * rsqrt_approx(q);
  }
  return __powf(sc, -beta);
}
template <bool B34>
__device__ __forceinline__ void lrn_pow2(float sc, float beta, float& sb, float& sb1) {
  if (B34) {
    const float q = rsqrt_approx(sc);
    const float q2 = q * q;
    sb = q2 * rsqrt_approx(q);
    sb1 = sb * q2;
  } else {
    sb = __powf(sc, -beta);
    sb1 = __fdividef(sb, sc);
  }
}

// Channel pairs (2m, 2m + 1) as float2, so that Blackwell's paired fp32
// instructions (__fadd2_rn, __fmul2_rn, __ffma2_rn) do two channels at once.
__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}
__device__ __forceinline__ void unpack4x2(const uint4& u, float2 (&p)[4]) {
  p[0] = bf2_to_f2(u.x);
  p[1] = bf2_to_f2(u.y);
  p[2] = bf2_to_f2(u.z);
  p[3] = bf2_to_f2(u.w);
}
__device__ __forceinline__ uint32_t f2_to_bf2(float2 v) {
  __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Sums over the five-channel window i - 2 .. i + 2 of the eight channels of
// a unit, from channel pairs P[0] = (c - 2, c - 1), P[1..4] = the unit's
// pairs, P[5] = (c + 8, c + 9).  With T_q = P[q].x + P[q].y, the window of
// channel 2m is T_{m} + T_{m+1} + P[m+2].x and that of 2m + 1 is
// P[m].y + T_{m+1} + T_{m+2} (pair indices of P).
__device__ __forceinline__ void window5(const float2 (&P)[6], float2 (&out)[4]) {
  float T[6];
#pragma unroll
  for (int q = 0; q < 6; ++q) T[q] = P[q].x + P[q].y;
#pragma unroll
  for (int m = 0; m < 4; ++m)
    out[m] = __fadd2_rn(__fadd2_rn(make_float2(T[m], P[m].y), make_float2(T[m + 1], T[m + 1])),
                        make_float2(P[m + 2].x, T[m + 2]));
}

// s^-beta and s^-beta-1 of a pair of normalisation scales (see lrn_pow2).
template <bool B34>
__device__ __forceinline__ void lrn_pow2x2(float2 sc, float beta, float2& sb, float2& sb1) {
  if (B34) {
    const float2 q = make_float2(rsqrt_approx(sc.x), rsqrt_approx(sc.y));
    const float2 q2 = __fmul2_rn(q, q);
    sb = __fmul2_rn(q2, make_float2(rsqrt_approx(q.x), rsqrt_approx(q.y)));
    sb1 = __fmul2_rn(sb, q2);
  } else {
    sb = make_float2(__powf(sc.x, -beta), __powf(sc.y, -beta));
    sb1 = make_float2(__fdividef(sb.x, sc.x), __fdividef(sb.y, sc.y));
  }
}

// Normalised values of a unit's eight channels ([S] 3.4 "Local Response
// Normalization": b_i = a_i (k + alpha sum_{|j - i| <= 2} a_j^2)^-beta), from
// channel pairs P[0] = (c - 2, c - 1), P[1..4] = the unit, P[5] =
// (c + 8, c + 9) (zeros outside the layer), packed to bf16.  Shared by the
// single normalisation kernel and the fused normalisation + pooling one, so
// the two give bit-identical maps.
template <bool B34>
__device__ __forceinline__ uint4 lrn8(const float2 (&P)[6], float2 k2, float2 alpha2, float beta) {
  float2 sq[6], S[4];
#pragma unroll
  for (int q = 0; q < 6; ++q) sq[q] = __fmul2_rn(P[q], P[q]);
  window5(sq, S);
  uint4 out;
  uint32_t* w = &out.x;
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float2 sb, sb1;
    lrn_pow2x2<B34>(__ffma2_rn(alpha2, S[m], k2), beta, sb, sb1);
    w[m] = f2_to_bf2(__fmul2_rn(P[1 + m], sb));
  }
  return out;
}

// ------------------------------------------------------------------ hparams
__global__ void k_write_hparams(HParams* hp, HParams v) { *hp = v; }

// ------------------------------------------------------------------ s2d
// One block per (image, pair of output rows i0, i0 + 1): the eight input
// rows 4 i0 .. 4 i0 + 7 are staged in shared memory, each at a stride of 688
// elements (rows past 226 and columns past 226 zero).  Output pixel j of row
// i holds channel (dy * 4 + dx) * 3 + c = x[4i + dy][4j + dx][c]: its
// channels 0-23 are the 12 elements at 12j of staged rows 4(i - i0) and
// 4(i - i0) + 1, channels 24-47 those of the next two rows, channels 48-63
// zero.  A thread writes one of these three parts of a pixel: six 8-byte
// shared loads, then 16-byte stores.
constexpr int kS2dRows = 2;  // output rows per block
__global__ void __launch_bounds__(256) k_s2d(const bf16* __restrict__ x, bf16* __restrict__ xs,
                                             int B) {
  constexpr int kRow = 227 * 3;  // elements per input row
  constexpr int kStride = 688;   // staged row stride: 8-byte aligned pixel groups
  constexpr int kIn = 4 * kS2dRows;
  constexpr int kWords = (kIn * kRow + 7) / 8 + 1;  // 16-byte words a block's rows can touch
  constexpr int kPer = (kWords + 255) / 256;
  __shared__ __align__(16) uint16_t st[kIn * kStride];
  const int tiles = (57 + kS2dRows - 1) / kS2dRows;
  const int i0 = (blockIdx.x % tiles) * kS2dRows;
  const int b = blockIdx.x / tiles;
  const int rows = min(kIn, 227 - 4 * i0);
  // the block's input rows are one contiguous run of rows * kRow elements;
  // it is read in 16-byte words aligned to x (x is 16-byte aligned), all of
  // a thread's words in flight at once, each word's in-range elements then
  // scattered to their staged row and column
  const long long base = (static_cast<long long>(b) * 227 + 4 * i0) * kRow;
  const int len = rows * kRow;
  const long long total = static_cast<long long>(B) * 227 * kRow;
  const long long w0 = base >> 3;
  const int lead = static_cast<int>(base - w0 * 8);  // elements of word 0 before the run
  // zero what no input element lands on: columns 681-687 of every staged
  // row, and the rows past the image
  for (int e = threadIdx.x; e < kIn * 8; e += blockDim.x) {
    const int r = e >> 3, c = kRow + (e & 7);
    if (c < kStride) st[r * kStride + c] = 0;
  }
  for (int e = threadIdx.x; e < (kIn - rows) * kStride; e += blockDim.x) st[rows * kStride + e] = 0;
  uint4 u[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const long long w = w0 + threadIdx.x + k * 256;
    u[k] = make_uint4(0, 0, 0, 0);
    if (w * 8 >= base + len) continue;
    if (w * 8 + 8 <= total) {
      u[k] = reinterpret_cast<const uint4*>(x)[w];
    } else {  // the tensor's last, partial word
      const uint16_t* xv = reinterpret_cast<const uint16_t*>(x);
      uint32_t h[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) h[q] = w * 8 + q < total ? xv[w * 8 + q] : 0u;
      u[k] = make_uint4(h[0] | h[1] << 16, h[2] | h[3] << 16, h[4] | h[5] << 16, h[6] | h[7] << 16);
    }
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int r0 = (threadIdx.x + k * 256) * 8 - lead;  // run index of the word's first element
    const uint32_t wv[4] = {u[k].x, u[k].y, u[k].z, u[k].w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int g = r0 + q;
      if (g >= 0 && g < len) {
        const int dy = g / kRow;
        st[dy * kStride + (g - dy * kRow)] =
            static_cast<uint16_t>(q & 1 ? wv[q >> 1] >> 16 : wv[q >> 1] & 0xFFFFu);
      }
    }
  }
  __syncthreads();
  const int nout = min(kS2dRows, 57 - i0);
  for (int t = threadIdx.x; t < nout * 57 * 3; t += blockDim.x) {
    const int ii = t / (57 * 3);
    const int u3 = t - ii * (57 * 3);
    const int j = u3 / 3, h = u3 - j * 3;
    uint4* o = reinterpret_cast<uint4*>(xs + ((static_cast<size_t>(b) * 57 + i0 + ii) * 57 + j) * 64) +
               h * 3;  // 16-byte chunks: 0-2, 3-5, 6-7
    if (h == 2) {
      o[0] = make_uint4(0, 0, 0, 0);
      o[1] = make_uint4(0, 0, 0, 0);
      continue;
    }
    const uint16_t* sr = st + (4 * ii + 2 * h) * kStride + 12 * j;
    const uint2* r0 = reinterpret_cast<const uint2*>(sr);
    const uint2* r1 = reinterpret_cast<const uint2*>(sr + kStride);
    const uint2 a0 = r0[0], a1 = r0[1], a2 = r0[2];
    const uint2 b0 = r1[0], b1 = r1[1], b2 = r1[2];
    o[0] = make_uint4(a0.x, a0.y, a1.x, a1.y);
    o[1] = make_uint4(a2.x, a2.y, b0.x, b0.y);
    o[2] = make_uint4(b1.x, b1.y, b2.x, b2.y);
  }
}

// ------------------------------------------------------------------ LRN
// [S] 3.4 "Local Response Normalization": b_i = a_i / (k + alpha * sum_{|j-i|<=2} a_j^2)^beta
// with the window clipped to the layer's channels (n = 5).
// Each thread owns one 8-channel chunk; consecutive lanes own consecutive
// chunks, so the channel halo comes from the neighbouring lanes (explicit
// loads only at the warp's edges).
template <bool B34>
__global__ void k_lrn_fwd(const bf16* __restrict__ a, bf16* __restrict__ b, long long P, int C,
                          float k, float alpha, float beta) {
  const uint32_t chunks = static_cast<uint32_t>(C) >> 3;
  const uint32_t n = static_cast<uint32_t>(P) * chunks;
  const int lane = threadIdx.x & 31;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; __any_sync(0xffffffffu, t < n);
       t += stride) {
    const bool active = t < n;
    const uint32_t p = active ? t / chunks : 0;
    const int c0 = active ? static_cast<int>(t - p * chunks) * 8 : 0;
    const bf16* ap = a + static_cast<size_t>(p) * C;
    float f[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) unpack8(*reinterpret_cast<const uint4*>(ap + c0), f);
    float2 P[6];
#pragma unroll
    for (int m = 0; m < 4; ++m) P[1 + m] = make_float2(f[2 * m], f[2 * m + 1]);
    const float up6 = __shfl_up_sync(0xffffffffu, f[6], 1), up7 = __shfl_up_sync(0xffffffffu, f[7], 1);
    const float dn0 = __shfl_down_sync(0xffffffffu, f[0], 1), dn1 = __shfl_down_sync(0xffffffffu, f[1], 1);
    P[0] = P[5] = make_float2(0.f, 0.f);
    if (active && c0 > 0) P[0] = lane > 0 ? make_float2(up6, up7) : ld_bf16x2(ap + c0 - 2);
    if (active && c0 + 8 < C) P[5] = lane < 31 ? make_float2(dn0, dn1) : ld_bf16x2(ap + c0 + 8);
    if (!active) continue;
    *reinterpret_cast<uint4*>(b + static_cast<size_t>(p) * C + c0) =
        lrn8<B34>(P, make_float2(k, k), make_float2(alpha, alpha), beta);
  }
}

// Backward: da_j = g_j s_j^-beta - 2 alpha beta a_j sum_{|i-j|<=2} g_i a_i s_i^(-beta-1),
// then times relu'(a_j) (a is the ReLU output, so a_j > 0 <=> the unit was active).
template <bool B34>
__global__ void k_lrn_bwd(const bf16* __restrict__ a, const bf16* __restrict__ g,
                          bf16* __restrict__ da, long long P, int C, float k, float alpha,
                          float beta) {
  const uint32_t chunks = static_cast<uint32_t>(C) >> 3;
  const uint32_t n = static_cast<uint32_t>(P) * chunks;
  const int lane = threadIdx.x & 31;
  const uint32_t stride = gridDim.x * blockDim.x;
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; __any_sync(0xffffffffu, t < n);
       t += stride) {
    const bool active = t < n;
    const uint32_t p = active ? t / chunks : 0;
    const int c0 = active ? static_cast<int>(t - p * chunks) * 8 : 0;
    const bf16* ap = a + static_cast<size_t>(p) * C;
    const bf16* gp = g + static_cast<size_t>(p) * C;
    float fa[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float fg[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (active) {
      unpack8(*reinterpret_cast<const uint4*>(ap + c0), fa);
      unpack8(*reinterpret_cast<const uint4*>(gp + c0), fg);
    }
    float av[16];  // channels c0-4 .. c0+11
    float gv[12];  // channels c0-2 .. c0+9
#pragma unroll
    for (int i = 0; i < 16; ++i) av[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 12; ++i) gv[i] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      av[4 + i] = fa[i];
      gv[2 + i] = fg[i];
    }
    float ua[4], ug[2], da_[4], dg[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ua[i] = __shfl_up_sync(0xffffffffu, fa[4 + i], 1);
      da_[i] = __shfl_down_sync(0xffffffffu, fa[i], 1);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      ug[i] = __shfl_up_sync(0xffffffffu, fg[6 + i], 1);
      dg[i] = __shfl_down_sync(0xffffffffu, fg[i], 1);
    }
    if (active && c0 > 0) {
      if (lane > 0) {
#pragma unroll
        for (int i = 0; i < 4; ++i) av[i] = ua[i];
        gv[0] = ug[0];
        gv[1] = ug[1];
      } else {
        const float2 a0 = ld_bf16x2(ap + c0 - 4), a1 = ld_bf16x2(ap + c0 - 2);
        av[0] = a0.x; av[1] = a0.y; av[2] = a1.x; av[3] = a1.y;
        const float2 g1 = ld_bf16x2(gp + c0 - 2);
        gv[0] = g1.x; gv[1] = g1.y;
      }
    }
    if (active && c0 + 8 < C) {
      if (lane < 31) {
#pragma unroll
        for (int i = 0; i < 4; ++i) av[12 + i] = da_[i];
        gv[10] = dg[0];
        gv[11] = dg[1];
      } else {
        const float2 a0 = ld_bf16x2(ap + c0 + 8), a1 = ld_bf16x2(ap + c0 + 10);
        av[12] = a0.x; av[13] = a0.y; av[14] = a1.x; av[15] = a1.y;
        const float2 g1 = ld_bf16x2(gp + c0 + 8);
        gv[10] = g1.x; gv[11] = g1.y;
      }
    }
    if (!active) continue;
    // s_i and t_i = g_i a_i s_i^(-beta-1) for channels c0-2 .. c0+9 (index i+2 in av)
    float sp[12], tt[12];
#pragma unroll
    for (int i = 0; i < 12; ++i) {
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < 5; ++j) sum += av[i + j] * av[i + j];
      const float sc = k + alpha * sum;
      float sb, sb1;
      lrn_pow2<B34>(sc, beta, sb, sb1);
      sp[i] = sb;
      tt[i] = gv[i] * av[i + 2] * sb1;
    }
    float o[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float cross = 0.f;
#pragma unroll
      for (int q = 0; q < 5; ++q) cross += tt[j + q];
      const float aj = av[j + 4];
      const float d = gv[j + 2] * sp[j + 2] - 2.f * alpha * beta * aj * cross;
      o[j] = aj > 0.f ? d : 0.f;
    }
    *reinterpret_cast<uint4*>(da + static_cast<size_t>(p) * C + c0) = pack8(o);
  }
}

__global__ void k_lrn_fwd_f32(const float* __restrict__ a, float* __restrict__ b, long long P,
                              int C, float k, float alpha, float beta) {
  const long long n = P * C;
  for (long long t = blockIdx.x * 1LL * blockDim.x + threadIdx.x; t < n;
       t += 1LL * gridDim.x * blockDim.x) {
    const long long p = t / C;
    const int c = static_cast<int>(t - p * C);
    const float* ap = a + p * C;
    float sum = 0.f;
    for (int j = max(0, c - 2); j <= min(C - 1, c + 2); ++j) sum += ap[j] * ap[j];
    b[t] = ap[c] * powf(k + alpha * sum, -beta);
  }
}

// ------------------------------------------------------------------ pooling
// [S] 3.4 "Overlapping Pooling": max over z x z windows at stride st, no padding.
template <int Z>
__global__ void k_pool_fwd(const bf16* __restrict__ x, bf16* __restrict__ y,
                           uint8_t* __restrict__ am, int B, int H, int W, int C, int st) {
  constexpr int z = Z;
  const uint32_t Ho = (H - z) / st + 1, Wo = (W - z) / st + 1;
  const uint32_t chunks = static_cast<uint32_t>(C) >> 3;
  const uint32_t n = static_cast<uint32_t>(B) * Ho * Wo * chunks;
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
    const uint32_t pix = t / chunks;
    const int c0 = static_cast<int>(t - pix * chunks) * 8;
    const uint32_t ow = pix % Wo;
    const uint32_t q = pix / Wo;
    const uint32_t oh = q % Ho;
    const uint32_t b = q / Ho;
    float best[8];
    int arg[8];
    const bf16* xb = x + (static_cast<size_t>(b * H + oh * st) * W + ow * st) * C + c0;
    uint4 win[Z * Z];
#pragma unroll
    for (int q = 0; q < Z * Z; ++q)
      win[q] = *reinterpret_cast<const uint4*>(xb + (static_cast<size_t>(q / Z) * W + q % Z) * C);
#pragma unroll
    for (int dy = 0; dy < z; ++dy)
#pragma unroll
      for (int dx = 0; dx < z; ++dx) {
        float f[8];
        unpack8(win[dy * Z + dx], f);
        const int off = dy * z + dx;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (off == 0 || f[i] > best[i]) {
            best[i] = f[i];
            arg[i] = off;
          }
        }
      }
    *reinterpret_cast<uint4*>(y + static_cast<size_t>(pix) * C + c0) = pack8(best);
    uint2 packed;
    packed.x = arg[0] | (arg[1] << 8) | (arg[2] << 16) | (arg[3] << 24);
    packed.y = arg[4] | (arg[5] << 8) | (arg[6] << 16) | (arg[7] << 24);
    *reinterpret_cast<uint2*>(am + static_cast<size_t>(pix) * C + c0) = packed;
  }
}

// bias_part (nullable; needs 256 % (C / 8) == 0 and 256 threads): per-block
// column sums of the stored dx, [gridDim.x][C] fp32.  A thread keeps the
// same 8 channels on every grid-stride step, so it sums them in registers.
__global__ void __launch_bounds__(256) k_pool_bwd(const bf16* __restrict__ dy,
                                                  const uint8_t* __restrict__ am,
                                                  const bf16* __restrict__ pooled,
                                                  bf16* __restrict__ dx, int B, int H, int W,
                                                  int C, int z, int st, int relu_mask,
                                                  float* __restrict__ bias_part) {
  const int Ho = (H - z) / st + 1, Wo = (W - z) / st + 1;
  const uint32_t chunks = static_cast<uint32_t>(C) >> 3;
  const uint32_t n = static_cast<uint32_t>(B) * H * W * chunks;
  float bsum[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (uint32_t t = blockIdx.x * blockDim.x + threadIdx.x; t < n; t += gridDim.x * blockDim.x) {
    const uint32_t pix = t / chunks;
    const int c0 = static_cast<int>(t - pix * chunks) * 8;
    const int iw = static_cast<int>(pix % W);
    const uint32_t q = pix / W;
    const int ih = static_cast<int>(q % H);
    const int b = static_cast<int>(q / H);
    const int oh_lo = ih < z ? 0 : (ih - z + st) / st;
    const int oh_hi = min(Ho - 1, ih / st);
    const int ow_lo = iw < z ? 0 : (iw - z + st) / st;
    const int ow_hi = min(Wo - 1, iw / st);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int oh = oh_lo; oh <= oh_hi; ++oh)
      for (int ow = ow_lo; ow <= ow_hi; ++ow) {
        const size_t o = (static_cast<size_t>(b * Ho + oh) * Wo + ow) * C + c0;
        const int off = (ih - oh * st) * z + (iw - ow * st);
        const uint2 a2 = *reinterpret_cast<const uint2*>(am + o);
        float g[8];
        unpack8(*reinterpret_cast<const uint4*>(dy + o), g);
        float pv[8];
        if (relu_mask) {
          unpack8(*reinterpret_cast<const uint4*>(pooled + o), pv);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) pv[i] = 1.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t word = i < 4 ? a2.x : a2.y;
          const int ai = (word >> (8 * (i & 3))) & 0xFF;
          if (ai == off && pv[i] > 0.f) acc[i] += g[i];
        }
      }
    const uint4 packed = pack8(acc);
    *reinterpret_cast<uint4*>(dx + static_cast<size_t>(pix) * C + c0) = packed;
    if (bias_part) {
      float r[8];
      unpack8(packed, r);
#pragma unroll
      for (int i = 0; i < 8; ++i) bsum[i] += r[i];
    }
  }
  if (!bias_part) return;
  // threads with the same channels (tid mod chunks) summed in thread order
  __shared__ float red[256 * 8];
  const int ch = static_cast<int>(threadIdx.x % chunks);
  const int grp = static_cast<int>(threadIdx.x / chunks);
#pragma unroll
  for (int i = 0; i < 8; ++i) red[grp * C + ch * 8 + i] = bsum[i];
  __syncthreads();
  const int groups = static_cast<int>(blockDim.x / chunks);
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float v = 0.f;
    for (int q = 0; q < groups; ++q) v += red[q * C + c];
    bias_part[static_cast<size_t>(blockIdx.x) * C + c] = v;
  }
}

// ------------------------------------------------------------------ LRN + pool
// Response normalisation followed by overlapping max-pooling ("ImageNet
// Classification with Deep Convolutional Neural Networks", 3.4 "Local
// Response Normalization" and "Overlapping Pooling"; the two follow the first
// and second convolutions in that order), fused: a block normalises the input
// rows under kPoolTileRows output rows of one image and one 32-channel slab
// into shared memory (rounded to bf16, the value a separate normalisation
// kernel would store), then pools them.  The normalised map reaches global
// memory only when `lo` is given.  Arithmetic and tie rule are those of
// k_lrn_fwd and k_pool_fwd.
constexpr int kPoolTileRows = 4;
constexpr int kSlab = 32;  // channels per block

// WC != 0: the map is WC x WC (H == W == WC known at compile time, so the
// index divisions are by constants).
template <int Z, int WC, bool B34>
__global__ void __launch_bounds__(256) k_lrn_pool_fwd(const bf16* __restrict__ a,
                                                      bf16* __restrict__ lo,
                                                      bf16* __restrict__ y,
                                                      uint8_t* __restrict__ am, int H_, int W_,
                                                      int C, float k, float alpha, float beta) {
  const int H = WC ? WC : H_, W = WC ? WC : W_;
  extern __shared__ __align__(16) uint4 lds[];  // [rows][W][4 chunks]
  const int Ho = (H - Z) / 2 + 1, Wo = (W - Z) / 2 + 1;
  // the channel slab varies fastest across the grid, so the blocks that
  // read a pixel's neighbouring slabs (the normalisation's channel halo
  // reaches into them) run together and share those lines in L2
  const int oh0 = blockIdx.y * kPoolTileRows;
  const int oh1 = min(Ho, oh0 + kPoolTileRows);
  const int b = blockIdx.z;
  const int cs = blockIdx.x * kSlab;
  const int r0 = 2 * oh0;
  // rows this block normalises: those its windows read; the last tile also
  // takes the rows below the last window so that `lo` is complete
  const int r1 = oh1 == Ho ? H : 2 * (oh1 - 1) + Z;
  // rows whose normalised values this block writes to `lo` (each row once)
  const int own1 = oh1 == Ho ? H : 2 * oh1;
  const int units1 = (r1 - r0) * W * 4;
  // four units per thread per pass, their loads issued before any is used
  constexpr int U = 4;
  for (int u0 = threadIdx.x; u0 < units1; u0 += U * blockDim.x) {
    uint4 v[U];
    uint32_t hl[U], hr[U];
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const int u = u0 + q * blockDim.x;
      v[q] = make_uint4(0, 0, 0, 0);
      hl[q] = hr[q] = 0;
      if (u < units1) {
        const int j = u & 3;
        const int x = (u >> 2) % W;
        const int r = (u >> 2) / W;
        const int c0 = cs + j * 8;
        const bf16* ap = a + ((static_cast<size_t>(b) * H + r0 + r) * W + x) * C + c0;
        v[q] = *reinterpret_cast<const uint4*>(ap);
        if (c0 > 0) hl[q] = *reinterpret_cast<const uint32_t*>(ap - 2);
        if (c0 + 8 < C) hr[q] = *reinterpret_cast<const uint32_t*>(ap + 8);
      }
    }
#pragma unroll
    for (int q = 0; q < U; ++q) {
      const int u = u0 + q * blockDim.x;
      if (u >= units1) break;
      const int j = u & 3;
      const int x = (u >> 2) % W;
      const int r = (u >> 2) / W;
      const int c0 = cs + j * 8;
      float2 P[6], mid[4];
      unpack4x2(v[q], mid);
#pragma unroll
      for (int m = 0; m < 4; ++m) P[1 + m] = mid[m];
      P[0] = bf2_to_f2(hl[q]);
      P[5] = bf2_to_f2(hr[q]);
      const uint4 packed = lrn8<B34>(P, make_float2(k, k), make_float2(alpha, alpha), beta);
      lds[(r * W + x) * 4 + j] = packed;
      if (lo && r0 + r < own1)
        *reinterpret_cast<uint4*>(lo + ((static_cast<size_t>(b) * H + r0 + r) * W + x) * C + c0) =
            packed;
    }
  }
  __syncthreads();
  const int units2 = (oh1 - oh0) * Wo * 4;
  for (int u = threadIdx.x; u < units2; u += blockDim.x) {
    const int j = u & 3;
    const int ow = (u >> 2) % Wo;
    const int oh = oh0 + (u >> 2) / Wo;
    // two channels per 32-bit word: values compared as bf16 pairs, the
    // window offset of each half's first maximum kept in the matching half
    uint32_t best[4], arg[4];
#pragma unroll
    for (int dy = 0; dy < Z; ++dy)
#pragma unroll
      for (int dx = 0; dx < Z; ++dx) {
        const uint4 w = lds[((2 * oh + dy - r0) * W + 2 * ow + dx) * 4 + j];
        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
        const uint32_t off = static_cast<uint32_t>(dy * Z + dx) * 0x00010001u;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (dy == 0 && dx == 0) {
            best[q] = wv[q];
            arg[q] = 0;
          } else {
            const uint32_t gt =
                __hgt2_mask(*reinterpret_cast<const __nv_bfloat162*>(&wv[q]),
                            *reinterpret_cast<const __nv_bfloat162*>(&best[q]));
            best[q] = (best[q] & ~gt) | (wv[q] & gt);
            arg[q] = (arg[q] & ~gt) | (off & gt);
          }
        }
      }
    const size_t o = ((static_cast<size_t>(b) * Ho + oh) * Wo + ow) * C + cs + j * 8;
    *reinterpret_cast<uint4*>(y + o) = make_uint4(best[0], best[1], best[2], best[3]);
    uint2 packed;  // one byte per channel: halves (lo, hi) of words 0..3
    packed.x = __byte_perm(arg[0], arg[1], 0x6420);
    packed.y = __byte_perm(arg[2], arg[3], 0x6420);
    *reinterpret_cast<uint2*>(am + o) = packed;
  }
}

// The channels of one pooled-gradient vector (8 bf16 in dyv) whose recorded
// window offset (one byte each in amv) equals `off`, added to g in fp32.
// The offset test works on all eight bytes at once: xor with the offset
// replicated into every byte, a carry-free per-byte non-zero test
// ((b & 0x7f) + 0x7f <= 0xfe, so no carry crosses a byte), then
// sign-replicating byte permutes widen each byte's flag to its channel's 16
// bits; the gradient is kept where the flag is clear.
__device__ __forceinline__ void add_routed8(const uint4& dyv, const uint2& amv, uint32_t off,
                                            float2 (&g)[4]) {
  const uint32_t rep = off * 0x01010101u;
  const uint32_t x0 = amv.x ^ rep, x1 = amv.y ^ rep;
  const uint32_t n0 = ((x0 & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x0;
  const uint32_t n1 = ((x1 & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x1;
  const uint4 kept = make_uint4(dyv.x & ~prmt(n0, 0, 0x9988), dyv.y & ~prmt(n0, 0, 0xBBAA),
                                dyv.z & ~prmt(n1, 0, 0x9988), dyv.w & ~prmt(n1, 0, 0xBBAA));
  float2 f[4];
  unpack4x2(kept, f);
#pragma unroll
  for (int m = 0; m < 4; ++m) g[m] = __fadd2_rn(g[m], f[m]);
}

// Backward of normalisation + pooling, fused: the pooled gradient is routed
// to the chosen pixels and pushed through the normalisation (and the ReLU
// below it, by the stored conv output a > 0) in one pass; `dl` (the
// normalised map's gradient) is written only when given.
//
// A thread owns a 2 x 2 quad of pixels (rows 2qi, 2qi + 1, columns 2qj,
// 2qj + 1) and one 8-channel unit.  With stride 2 the windows that can
// route gradient into the quad are (qi - 1 + wr, qj - 1 + wc), wr, wc in
// {0, 1} (only (qi, qj) for z = 2), and the pixel at (h, d) of the quad sits
// at offset (h + 2 - 2 wr, d + 2 - 2 wc) of window (wr, wc): the four windows
// are loaded once for four pixels, and which pixel may take which window is
// known at compile time.  Gradients are summed in ascending (row-major)
// window order.  The normalisation's channel window reaches two channels
// into the neighbouring units; those edge values (a, then the cross terms
// t_i = g_i a_i s_i^(-beta-1)) go through shared memory, one quad row at a
// time.  The arithmetic works on channel pairs with paired fp32
// instructions.  Per block the column sums of the stored da (the layer's
// bias gradient) are written to bias_part[blockIdx.x][C] (nullable).
template <int ZC, int WC, bool B34>
__global__ void __launch_bounds__(256) k_pool_lrn_bwd(const bf16* __restrict__ dy,
                                                      const uint8_t* __restrict__ am,
                                                      const bf16* __restrict__ a,
                                                      bf16* __restrict__ dl,
                                                      bf16* __restrict__ da, int nquads,
                                                      int nq, int H_, int W_, int C, int z_,
                                                      float k, float alpha, float beta,
                                                      float* __restrict__ bias_part) {
  // ZC / WC != 0: window and (square) map size known at compile time
  const int H = WC ? WC : H_, W = WC ? WC : W_, z = ZC ? ZC : z_;
  const int Ho = (H - z) / 2 + 1, Wo = (W - z) / 2 + 1;
  const int QH = (H + 1) >> 1, QW = (W + 1) >> 1;
  const int CH = C >> 3;
  const int up = threadIdx.x / CH;
  const int uj = threadIdx.x - up * CH;
  const bool mine = up < nq;
  const int tid = threadIdx.x;
  // edge pairs of every thread's unit (channels 0, 1 and 6, 7), per quad
  // column: normalisation inputs (ea) and cross terms (et)
  __shared__ float4 ea[2][256], et[2][256];
  __shared__ float red[256 * 8];
  const float2 k2 = make_float2(k, k), alpha2 = make_float2(alpha, alpha);
  const float2 mc2ab = make_float2(-2.f * alpha * beta, -2.f * alpha * beta);
  float2 bsum[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) bsum[m] = make_float2(0.f, 0.f);
  for (int blk = blockIdx.x; blk * nq < nquads; blk += gridDim.x) {
    const int q = blk * nq + up;
    const bool live = mine && q < nquads;
    int b = 0, qi = 0, qj = 0;
    if (live) {
      qj = q % QW;
      const int r = q / QW;
      qi = r % QH;
      b = r / QH;
    }
    uint4 wdy[4];
    uint2 wam[4];
    bool wok[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int oh = qi - 1 + (w >> 1), ow = qj - 1 + (w & 1);
      wok[w] = live && oh >= 0 && oh < Ho && ow >= 0 && ow < Wo && (z == 3 || w == 3);
      wdy[w] = make_uint4(0, 0, 0, 0);
      wam[w] = make_uint2(0, 0);
      if (wok[w]) {
        const uint32_t o = static_cast<uint32_t>((b * Ho + oh) * Wo + ow) * C + uj * 8;
        wdy[w] = *reinterpret_cast<const uint4*>(dy + o);
        wam[w] = *reinterpret_cast<const uint2*>(am + o);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ih = 2 * qi + h;
      float2 g[2][4], av[2][4];
      bool pv[2];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const int iw = 2 * qj + d;
        pv[d] = live && ih < H && iw < W;
#pragma unroll
        for (int m = 0; m < 4; ++m) g[d][m] = av[d][m] = make_float2(0.f, 0.f);
        if (pv[d]) {
          unpack4x2(*reinterpret_cast<const uint4*>(
                        a + static_cast<uint32_t>((b * H + ih) * W + iw) * C + uj * 8),
                    av[d]);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int rr = h + 2 - 2 * (w >> 1), rc = d + 2 - 2 * (w & 1);
            if (wok[w] && rr < z && rc < z)
              add_routed8(wdy[w], wam[w], static_cast<uint32_t>(rr * z + rc), g[d]);
          }
        }
        ea[d][tid] = make_float4(av[d][0].x, av[d][0].y, av[d][3].x, av[d][3].y);
      }
      __syncthreads();
      float2 first[2][4], tv[2][4];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const float4 L = mine && uj > 0 ? ea[d][tid - 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 R = mine && uj < CH - 1 ? ea[d][tid + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        float2 sq[6], S[4];
        sq[0] = __fmul2_rn(make_float2(L.z, L.w), make_float2(L.z, L.w));
#pragma unroll
        for (int m = 0; m < 4; ++m) sq[1 + m] = __fmul2_rn(av[d][m], av[d][m]);
        sq[5] = __fmul2_rn(make_float2(R.x, R.y), make_float2(R.x, R.y));
        window5(sq, S);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float2 sb, sb1;
          lrn_pow2x2<B34>(__ffma2_rn(alpha2, S[m], k2), beta, sb, sb1);
          first[d][m] = __fmul2_rn(g[d][m], sb);
          tv[d][m] = __fmul2_rn(__fmul2_rn(g[d][m], av[d][m]), sb1);
        }
        et[d][tid] = make_float4(tv[d][0].x, tv[d][0].y, tv[d][3].x, tv[d][3].y);
      }
      __syncthreads();
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const float4 L = mine && uj > 0 ? et[d][tid - 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 R = mine && uj < CH - 1 ? et[d][tid + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
        if (!pv[d]) continue;
        float2 tp[6], cross[4];
        tp[0] = make_float2(L.z, L.w);
#pragma unroll
        for (int m = 0; m < 4; ++m) tp[1 + m] = tv[d][m];
        tp[5] = make_float2(R.x, R.y);
        window5(tp, cross);
        uint4 packed;
        uint32_t* pw = &packed.x;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float2 dd = __ffma2_rn(mc2ab, __fmul2_rn(av[d][m], cross[m]), first[d][m]);
          pw[m] = f2_to_bf2(make_float2(av[d][m].x > 0.f ? dd.x : 0.f,
                                        av[d][m].y > 0.f ? dd.y : 0.f));
        }
        const uint32_t e = static_cast<uint32_t>((b * H + ih) * W + 2 * qj + d) * C + uj * 8;
        *reinterpret_cast<uint4*>(da + e) = packed;
        if (dl) {
          uint4 gp;
          gp.x = f2_to_bf2(g[d][0]);
          gp.y = f2_to_bf2(g[d][1]);
          gp.z = f2_to_bf2(g[d][2]);
          gp.w = f2_to_bf2(g[d][3]);
          *reinterpret_cast<uint4*>(dl + e) = gp;
        }
        float2 r[4];
        unpack4x2(packed, r);
#pragma unroll
        for (int m = 0; m < 4; ++m) bsum[m] = __fadd2_rn(bsum[m], r[m]);
      }
    }
  }
  if (!bias_part) return;
  // per-channel sum over the block's quad slots, in slot order
  if (mine) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      red[up * C + uj * 8 + 2 * m] = bsum[m].x;
      red[up * C + uj * 8 + 2 * m + 1] = bsum[m].y;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    float v = 0.f;
    for (int q = 0; q < nq; ++q) v += red[q * C + c];
    bias_part[static_cast<size_t>(blockIdx.x) * C + c] = v;
  }
}

// The same backward with each quad's CH = C / 8 channel units in
// consecutive lanes of one warp (32 / CH quads per warp; C <= 256): the
// normalisation's channel halo moves between neighbouring lanes by shuffles,
// so the loop needs no block-wide barrier and a warp never waits for
// another.  Lanes past the last whole quad of a warp stay idle.  Same
// arithmetic, window order and bias partial layout as k_pool_lrn_bwd.
template <int ZC, int WC, bool B34>
__global__ void __launch_bounds__(256, 3) k_pool_lrn_bwd_w(const bf16* __restrict__ dy,
                                                        const uint8_t* __restrict__ am,
                                                        const bf16* __restrict__ a,
                                                        bf16* __restrict__ dl,
                                                        bf16* __restrict__ da, int nquads,
                                                        int H_, int W_, int C, int z_, float k,
                                                        float alpha, float beta,
                                                        float* __restrict__ bias_part) {
  const int H = WC ? WC : H_, W = WC ? WC : W_, z = ZC ? ZC : z_;
  const int Ho = (H - z) / 2 + 1, Wo = (W - z) / 2 + 1;
  const int QH = (H + 1) >> 1, QW = (W + 1) >> 1;
  const int CH = C >> 3;
  const int qpw = 32 / CH;  // quads per warp
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int qslot = lane / CH, uj = lane - qslot * CH;
  const bool mine = qslot < qpw;
  const int wpb = blockDim.x >> 5;
  __shared__ float red[8 * 32 * 8];  // [warp][lane][8 channels]
  const float2 k2 = make_float2(k, k), alpha2 = make_float2(alpha, alpha);
  const float2 mc2ab = make_float2(-2.f * alpha * beta, -2.f * alpha * beta);
  float2 bsum[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) bsum[m] = make_float2(0.f, 0.f);
  const int gwarp = blockIdx.x * wpb + warp, nwarps = gridDim.x * wpb;
  for (int q0 = gwarp * qpw; q0 < nquads; q0 += nwarps * qpw) {
    const int q = q0 + qslot;
    const bool live = mine && q < nquads;
    int b = 0, qi = 0, qj = 0;
    if (live) {
      qj = q % QW;
      const int r = q / QW;
      qi = r % QH;
      b = r / QH;
    }
    uint4 wdy[4];
    uint2 wam[4];
    bool wok[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int oh = qi - 1 + (w >> 1), ow = qj - 1 + (w & 1);
      wok[w] = live && oh >= 0 && oh < Ho && ow >= 0 && ow < Wo && (z == 3 || w == 3);
      wdy[w] = make_uint4(0, 0, 0, 0);
      wam[w] = make_uint2(0, 0);
      if (wok[w]) {
        const uint32_t o = static_cast<uint32_t>((b * Ho + oh) * Wo + ow) * C + uj * 8;
        wdy[w] = *reinterpret_cast<const uint4*>(dy + o);
        wam[w] = *reinterpret_cast<const uint2*>(am + o);
      }
    }
#pragma unroll
    for (int px = 0; px < 4; ++px) {
      const int h = px >> 1, d = px & 1;
      const int ih = 2 * qi + h, iw = 2 * qj + d;
      const bool pv = live && ih < H && iw < W;
      float2 g[4], av[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) g[m] = av[m] = make_float2(0.f, 0.f);
      if (pv) {
        unpack4x2(*reinterpret_cast<const uint4*>(
                      a + static_cast<uint32_t>((b * H + ih) * W + iw) * C + uj * 8),
                  av);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int rr = h + 2 - 2 * (w >> 1), rc = d + 2 - 2 * (w & 1);
          if (wok[w] && rr < z && rc < z)
            add_routed8(wdy[w], wam[w], static_cast<uint32_t>(rr * z + rc), g);
        }
      }
      // channel halo from the neighbouring lanes of the same quad
      float2 Lh = make_float2(__shfl_up_sync(0xffffffffu, av[3].x, 1),
                              __shfl_up_sync(0xffffffffu, av[3].y, 1));
      float2 Rh = make_float2(__shfl_down_sync(0xffffffffu, av[0].x, 1),
                              __shfl_down_sync(0xffffffffu, av[0].y, 1));
      if (uj == 0) Lh = make_float2(0.f, 0.f);
      if (uj == CH - 1) Rh = make_float2(0.f, 0.f);
      float2 sq[6], S[4], first[4], tv[4];
      sq[0] = __fmul2_rn(Lh, Lh);
#pragma unroll
      for (int m = 0; m < 4; ++m) sq[1 + m] = __fmul2_rn(av[m], av[m]);
      sq[5] = __fmul2_rn(Rh, Rh);
      window5(sq, S);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float2 sb, sb1;
        lrn_pow2x2<B34>(__ffma2_rn(alpha2, S[m], k2), beta, sb, sb1);
        first[m] = __fmul2_rn(g[m], sb);
        tv[m] = __fmul2_rn(__fmul2_rn(g[m], av[m]), sb1);
      }
      float2 TL = make_float2(__shfl_up_sync(0xffffffffu, tv[3].x, 1),
                              __shfl_up_sync(0xffffffffu, tv[3].y, 1));
      float2 TR = make_float2(__shfl_down_sync(0xffffffffu, tv[0].x, 1),
                              __shfl_down_sync(0xffffffffu, tv[0].y, 1));
      if (uj == 0) TL = make_float2(0.f, 0.f);
      if (uj == CH - 1) TR = make_float2(0.f, 0.f);
      if (!pv) continue;
      float2 tp[6], cross[4];
      tp[0] = TL;
#pragma unroll
      for (int m = 0; m < 4; ++m) tp[1 + m] = tv[m];
      tp[5] = TR;
      window5(tp, cross);
      uint4 packed;
      uint32_t* pw = &packed.x;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float2 dd = __ffma2_rn(mc2ab, __fmul2_rn(av[m], cross[m]), first[m]);
        pw[m] = f2_to_bf2(make_float2(av[m].x > 0.f ? dd.x : 0.f, av[m].y > 0.f ? dd.y : 0.f));
      }
      const uint32_t e = static_cast<uint32_t>((b * H + ih) * W + iw) * C + uj * 8;
      *reinterpret_cast<uint4*>(da + e) = packed;
      if (dl) {
        uint4 gp;
        gp.x = f2_to_bf2(g[0]);
        gp.y = f2_to_bf2(g[1]);
        gp.z = f2_to_bf2(g[2]);
        gp.w = f2_to_bf2(g[3]);
        *reinterpret_cast<uint4*>(dl + e) = gp;
      }
      float2 r[4];
      unpack4x2(packed, r);
#pragma unroll
      for (int m = 0; m < 4; ++m) bsum[m] = __fadd2_rn(bsum[m], r[m]);
    }
  }
  if (!bias_part) return;
  // per-channel sums over the block's (warp, quad slot) pairs, in that order
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    red[(warp * 32 + lane) * 8 + 2 * m] = bsum[m].x;
    red[(warp * 32 + lane) * 8 + 2 * m + 1] = bsum[m].y;
  }
  __syncthreads();
  for (int c = threadIdx.x; c < C; c += blockDim.x) {
    const int u = c >> 3, i = c & 7;
    float v = 0.f;
    for (int w = 0; w < wpb; ++w)
      for (int qs = 0; qs < qpw; ++qs) v += red[(w * 32 + qs * CH + u) * 8 + i];
    bias_part[static_cast<size_t>(blockIdx.x) * C + c] = v;
  }
}

// The same backward with each work item's rows staged in shared memory by
// bulk asynchronous copies, so that the loads of the next items are in
// flight while one is computed.  Item (b, qi) = quad row qi of image b: the
// input rows 2 qi, 2 qi + 1 of a (contiguous in NHWC) and the pooled rows
// qi - 1, qi of dy and of the window choices (the only windows that cover
// the quad row).  Thread (qj, uj) = quad column qj, channel unit uj (eight
// channels), blockDim = QW * CH rounded up to a warp (at most 448, two
// blocks per SM); the channel halo of the normalisation sums is read from
// the staged row itself, that of the cross term goes through shared memory
// (two barriers per input row).  Every bulk copy lands in a stage no thread
// reads any more (a block barrier precedes the issue); every wait is
// bounded.  Per block, the column sums of the stored da go to
// bias_part[blockIdx.x][C] in a fixed order.
struct PlbGeom {
  int rowA, rowO;              // elements per input / pooled row
  int off_dy, off_am, stage;   // byte offsets within a stage, stage bytes
};
__host__ __device__ inline int round128(int v) { return (v + 127) & ~127; }
__host__ __device__ inline PlbGeom plb_geom(int W, int Wo, int C) {
  PlbGeom g;
  g.rowA = W * C;
  g.rowO = Wo * C;
  g.off_dy = round128(2 * g.rowA * 2);
  g.off_am = g.off_dy + round128(2 * g.rowO * 2);
  g.stage = g.off_am + round128(2 * g.rowO);
  return g;
}

// LRN = false: the same staged pool backward without a normalisation
// between the conv output and the pool (pool5, and the pages' no-LRN
// ablation): da = ReLU'(a) * (the routed pooled gradient).
template <int ZC, int WC, bool B34, bool LRN = true>
__global__ void __launch_bounds__(448, 2) k_pool_lrn_bwd_s(
    const bf16* __restrict__ dy, const uint8_t* __restrict__ am, const bf16* __restrict__ a,
    bf16* __restrict__ dl, bf16* __restrict__ da, int B, int H_, int W_, int C, int z_, float k,
    float alpha, float beta, int nst, float* __restrict__ bias_part, int* status) {
  const int H = WC ? WC : H_, W = WC ? WC : W_, z = ZC ? ZC : z_;
  const int Ho = (H - z) / 2 + 1, Wo = (W - z) / 2 + 1;
  const int QH = (H + 1) >> 1;
  const int QW = (W + 1) >> 1;
  const int CH = C >> 3;
  const PlbGeom G = plb_geom(W, Wo, C);
  extern __shared__ __align__(128) uint8_t plb_smem[];
  const int nt = blockDim.x;
  float4* tvs = reinterpret_cast<float4*>(plb_smem + nst * G.stage);  // [pixel][thread]
  uint64_t* bars = reinterpret_cast<uint64_t*>(tvs + 2 * nt);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + nst);
  const uint32_t bar0 = smem_u32(bars);
  const int tid = threadIdx.x;
  const int qj = tid / CH, uj = tid - qj * CH;
  const bool mine = qj < QW;
  const int items = B * QH;
  const float2 k2 = make_float2(k, k), alpha2 = make_float2(alpha, alpha);
  const float2 mc2ab = make_float2(-2.f * alpha * beta, -2.f * alpha * beta);

  // the pooled rows an item needs: qi - 1 (z = 3 only) .. qi, inside the map
  auto out_rows = [&](int qi, int& olo) {
    olo = z == 3 ? max(qi - 1, 0) : qi;
    const int ohi = min(qi, Ho - 1);
    return ohi >= olo ? ohi - olo + 1 : 0;
  };
  auto issue = [&](int item, int st) {
    const int b = item / QH, qi = item - b * QH;
    const int nra = min(2, H - 2 * qi);
    int olo;
    const int nro = out_rows(qi, olo);
    const uint32_t bar = bar0 + 8 * st;
    const uint32_t dst = smem_u32(plb_smem + st * G.stage);
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nra * G.rowA * 2 + nro * G.rowO * 3));
    bulk_load(dst, a + (static_cast<size_t>(b) * H + 2 * qi) * G.rowA,
              static_cast<uint32_t>(nra * G.rowA * 2), bar);
    if (nro) {
      const size_t o = (static_cast<size_t>(b) * Ho + olo) * G.rowO;
      bulk_load(dst + G.off_dy, dy + o, static_cast<uint32_t>(nro * G.rowO * 2), bar);
      bulk_load(dst + G.off_am, am + o, static_cast<uint32_t>(nro * G.rowO), bar);
    }
  };

  if (tid == 0) {
    for (int st = 0; st < nst; ++st) mbar_init(bar0 + 8 * st, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    for (int st = 0; st < nst; ++st) {
      const int item = blockIdx.x + st * gridDim.x;
      if (item < items) issue(item, st);
    }
  }

  float2 bsum[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) bsum[m] = make_float2(0.f, 0.f);
  int n = 0;
  bool aborted = false;
  for (int item = blockIdx.x; item < items; item += gridDim.x, ++n) {
    const int st = n % nst;
    // (a thread whose wait gave up computes on whatever the stage holds,
    // in bounds, and leaves with the others at the first barrier)
    mbar_wait_limit(bar0 + 8 * st, static_cast<uint32_t>((n / nst) & 1), status, abort_flag,
                     WAIT_LIMIT_CYCLES);
    const int b = item / QH, qi = item - b * QH;
    int olo;
    out_rows(qi, olo);
    const uint8_t* sbase = plb_smem + st * G.stage;
    const bf16* SA = reinterpret_cast<const bf16*>(sbase);
    const bf16* SD = reinterpret_cast<const bf16*>(sbase + G.off_dy);
    const uint8_t* SM = sbase + G.off_am;
    uint4 wdy[4];
    uint2 wam[4];
    bool wok[4];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int oh = qi - 1 + (w >> 1), ow = qj - 1 + (w & 1);
      wok[w] = mine && oh >= 0 && oh < Ho && ow >= 0 && ow < Wo && (z == 3 || w == 3);
      wdy[w] = make_uint4(0, 0, 0, 0);
      wam[w] = make_uint2(0, 0);
      if (wok[w]) {
        const int o = (oh - olo) * G.rowO + ow * C + uj * 8;
        wdy[w] = *reinterpret_cast<const uint4*>(SD + o);
        wam[w] = *reinterpret_cast<const uint2*>(SM + o);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ih = 2 * qi + h;
      float2 first[2][4], tv[2][4];
      bool pv[2];
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        const int iw = 2 * qj + d;
        pv[d] = mine && ih < H && iw < W;
        float2 g[4], P[6];
#pragma unroll
        for (int m = 0; m < 4; ++m) g[m] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 6; ++q) P[q] = make_float2(0.f, 0.f);
        if (pv[d]) {
          const int o = h * G.rowA + iw * C + uj * 8;
          if constexpr (LRN) {
            float2 av[4];
            unpack4x2(*reinterpret_cast<const uint4*>(SA + o), av);
#pragma unroll
            for (int m = 0; m < 4; ++m) P[1 + m] = av[m];
            if (uj > 0) P[0] = bf2_to_f2(*reinterpret_cast<const uint32_t*>(SA + o - 2));
            if (uj < CH - 1) P[5] = bf2_to_f2(*reinterpret_cast<const uint32_t*>(SA + o + 8));
          }
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            const int rr = h + 2 - 2 * (w >> 1), rc = d + 2 - 2 * (w & 1);
            if (wok[w] && rr < z && rc < z)
              add_routed8(wdy[w], wam[w], static_cast<uint32_t>(rr * z + rc), g);
          }
          if (dl) {
            uint4 gp;
            gp.x = f2_to_bf2(g[0]);
            gp.y = f2_to_bf2(g[1]);
            gp.z = f2_to_bf2(g[2]);
            gp.w = f2_to_bf2(g[3]);
            *reinterpret_cast<uint4*>(
                dl + static_cast<uint32_t>((b * H + ih) * W + iw) * C + uj * 8) = gp;
          }
        }
        if constexpr (LRN) {
          float2 sq[6], S[4];
#pragma unroll
          for (int q = 0; q < 6; ++q) sq[q] = __fmul2_rn(P[q], P[q]);
          window5(sq, S);
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            float2 sb, sb1;
            lrn_pow2x2<B34>(__ffma2_rn(alpha2, S[m], k2), beta, sb, sb1);
            first[d][m] = __fmul2_rn(g[m], sb);
            tv[d][m] = __fmul2_rn(__fmul2_rn(g[m], P[1 + m]), sb1);
          }
          tvs[d * nt + tid] = make_float4(tv[d][0].x, tv[d][0].y, tv[d][3].x, tv[d][3].y);
        } else {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            first[d][m] = g[m];
            tv[d][m] = make_float2(0.f, 0.f);
          }
        }
      }
      __syncthreads();
      if (*abort_flag) break;
#pragma unroll
      for (int d = 0; d < 2; ++d) {
        if (!pv[d]) continue;
        const int iw = 2 * qj + d;
        float2 av[4], cross[4];
        unpack4x2(*reinterpret_cast<const uint4*>(SA + h * G.rowA + iw * C + uj * 8), av);
        if constexpr (LRN) {
          const float4 L = uj > 0 ? tvs[d * nt + tid - 1] : make_float4(0.f, 0.f, 0.f, 0.f);
          const float4 R =
              uj < CH - 1 ? tvs[d * nt + tid + 1] : make_float4(0.f, 0.f, 0.f, 0.f);
          float2 tp[6];
          tp[0] = make_float2(L.z, L.w);
#pragma unroll
          for (int m = 0; m < 4; ++m) tp[1 + m] = tv[d][m];
          tp[5] = make_float2(R.x, R.y);
          window5(tp, cross);
        }
        uint4 packed;
        uint32_t* pw = &packed.x;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const float2 dd =
              LRN ? __ffma2_rn(mc2ab, __fmul2_rn(av[m], cross[m]), first[d][m]) : first[d][m];
          pw[m] = f2_to_bf2(make_float2(av[m].x > 0.f ? dd.x : 0.f, av[m].y > 0.f ? dd.y : 0.f));
        }
        *reinterpret_cast<uint4*>(da + static_cast<uint32_t>((b * H + ih) * W + iw) * C +
                                  uj * 8) = packed;
        float2 r[4];
        unpack4x2(packed, r);
#pragma unroll
        for (int m = 0; m < 4; ++m) bsum[m] = __fadd2_rn(bsum[m], r[m]);
      }
      // the cross-term slots are free again; after the second row, stage st too
      __syncthreads();
    }
    if (*abort_flag) {
      aborted = true;
      break;
    }
    if (tid == 0) {
      const int next = item + nst * gridDim.x;
      if (next < items) {
        fence_proxy_async_smem();
        issue(next, st);
      }
    }
  }
  if (aborted) {
    // copies still in flight land before the block exits (bounded wait)
    if (tid == 0) {
      for (int j = 0; j < nst; ++j) {
        const int nn = n + j;
        if (blockIdx.x + nn * gridDim.x >= items) break;
        const uint32_t bar = bar0 + 8 * (nn % nst);
        const uint32_t par = static_cast<uint32_t>((nn / nst) & 1);
        for (int i = 0; i < (1 << 20) && !mbar_try_wait(bar, par); ++i) __nanosleep(64);
      }
    }
    return;
  }
  if (!bias_part) return;
  // per-channel sums over the block's quad columns, in column order (the
  // stages are idle: every issued copy has been consumed)
  float* red = reinterpret_cast<float*>(plb_smem);
  if (mine) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      red[qj * C + uj * 8 + 2 * m] = bsum[m].x;
      red[qj * C + uj * 8 + 2 * m + 1] = bsum[m].y;
    }
  }
  __syncthreads();
  for (int c = tid; c < C; c += nt) {
    float v = 0.f;
    for (int q = 0; q < QW; ++q) v += red[q * C + c];
    bias_part[static_cast<size_t>(blockIdx.x) * C + c] = v;
  }
}

__global__ void k_pool_fwd_f32(const float* __restrict__ x, float* __restrict__ y, int B, int H,
                               int W, int C, int z, int st) {
  const int Ho = (H - z) / st + 1, Wo = (W - z) / st + 1;
  const long long n = 1LL * B * Ho * Wo * C;
  for (long long t = blockIdx.x * 1LL * blockDim.x + threadIdx.x; t < n;
       t += 1LL * gridDim.x * blockDim.x) {
    const int c = static_cast<int>(t % C);
    const long long pix = t / C;
    const int ow = static_cast<int>(pix % Wo);
    const int oh = static_cast<int>((pix / Wo) % Ho);
    const int b = static_cast<int>(pix / (1LL * Wo * Ho));
    float best = 0.f;
    for (int dy = 0; dy < z; ++dy)
      for (int dx = 0; dx < z; ++dx) {
        const float v = x[((1LL * b * H + oh * st + dy) * W + ow * st + dx) * C + c];
        if ((dy == 0 && dx == 0) || v > best) best = v;
      }
    y[t] = best;
  }
}

// ------------------------------------------------------------------ FC epilogues
// Dropout ([S] 3.4 "Dropout"): element e = row*cols + col of FC layer `layer`
// is kept iff word (e & 3) of Philox4x32-10((e >> 2, layer, step, 0),
// (seed_lo, seed_hi)) >= drop_thresh; kept units are not rescaled at
// training time; at inference every unit is multiplied by 1 - p.
__device__ __forceinline__ U4 dropout_words(const HParams& hp, long long e4, int layer) {
  U4 c{static_cast<uint32_t>(e4), static_cast<uint32_t>(layer), hp.step, 0u};
  return philox4x32_10(c, hp.seed_lo, hp.seed_hi);
}

__global__ void k_fc_finalize(const float* __restrict__ part, int S, int rows, int cols,
                              const float* __restrict__ bias, int relu, int dropout_mode,
                              int layer, const HParams* __restrict__ hpp, bf16* out_bf16,
                              float* out_f32) {
  const HParams hp = *hpp;
  const long long n4 = 1LL * rows * cols / 4;
  const long long plane = 1LL * rows * cols;
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n4;
       q += 1LL * gridDim.x * blockDim.x) {
    const long long e = q * 4;
    const int col = static_cast<int>(static_cast<uint32_t>(e) % static_cast<uint32_t>(cols));
    float4 acc = *reinterpret_cast<const float4*>(part + e);
    // slices added in order s = 1, 2, ...; four loads in flight
    int s = 1;
    for (; s + 4 <= S; s += 4) {
      float4 p[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) p[k] = *reinterpret_cast<const float4*>(part + (s + k) * plane + e);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc.x += p[k].x; acc.y += p[k].y; acc.z += p[k].z; acc.w += p[k].w;
      }
    }
    for (; s < S; ++s) {
      const float4 p = *reinterpret_cast<const float4*>(part + s * plane + e);
      acc.x += p.x; acc.y += p.y; acc.z += p.z; acc.w += p.w;
    }
    float v[4] = {acc.x, acc.y, acc.z, acc.w};
    if (bias) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] += bias[col + i];
    }
    if (relu) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = v[i] > 0.f ? v[i] : 0.f;
    }
    if (dropout_mode == 1) {
      const U4 w = dropout_words(hp, q + static_cast<long long>(hp.row_offset) * (cols / 4), layer);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = u4_word(w, i) >= hp.drop_thresh ? v[i] : 0.f;
    } else if (dropout_mode == 2) {
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= (1.f - hp.dropout_p);
    }
    if (out_bf16) {
      uint2 u;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(v[2], v[3]);
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(out_bf16 + e) = u;
    } else {
      *reinterpret_cast<float4*>(out_f32 + e) = make_float4(v[0], v[1], v[2], v[3]);
    }
  }
}

__global__ void k_dropout_mask(const HParams* __restrict__ hpp, int layer, int rows, int cols,
                               uint8_t* keep) {
  const HParams hp = *hpp;
  const long long n4 = 1LL * rows * cols / 4;
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n4;
       q += 1LL * gridDim.x * blockDim.x) {
    const U4 w = dropout_words(hp, q + static_cast<long long>(hp.row_offset) * (cols / 4), layer);
#pragma unroll
    for (int i = 0; i < 4; ++i) keep[q * 4 + i] = u4_word(w, i) >= hp.drop_thresh ? 1 : 0;
  }
}

__global__ void k_dgrad_finalize(const float* __restrict__ part, int S, int rows, int cols,
                                 const bf16* __restrict__ mask, bf16* __restrict__ out) {
  const long long n8 = 1LL * rows * cols / 8;
  const long long plane = 1LL * rows * cols;
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n8;
       q += 1LL * gridDim.x * blockDim.x) {
    const long long e = q * 8;
    float v[8];
    {
      const float4 a = *reinterpret_cast<const float4*>(part + e);
      const float4 b = *reinterpret_cast<const float4*>(part + e + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    // slices added in order s = 1, 2, ...; two slices (four loads) in flight
    int s = 1;
    for (; s + 2 <= S; s += 2) {
      float4 a[2], b[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        a[k] = *reinterpret_cast<const float4*>(part + (s + k) * plane + e);
        b[k] = *reinterpret_cast<const float4*>(part + (s + k) * plane + e + 4);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        v[0] += a[k].x; v[1] += a[k].y; v[2] += a[k].z; v[3] += a[k].w;
        v[4] += b[k].x; v[5] += b[k].y; v[6] += b[k].z; v[7] += b[k].w;
      }
    }
    for (; s < S; ++s) {
      const float4 a = *reinterpret_cast<const float4*>(part + s * plane + e);
      const float4 b = *reinterpret_cast<const float4*>(part + s * plane + e + 4);
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w;
      v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
    if (mask) {
      float m[8];
      unpack8(*reinterpret_cast<const uint4*>(mask + e), m);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = m[i] > 0.f ? v[i] : 0.f;
    }
    *reinterpret_cast<uint4*>(out + e) = pack8(v);
  }
}

// ------------------------------------------------------------------ softmax + CE
// [S] 3.4 "Training Procedure Details", "Objective function": the mean over
// the batch of -log softmax(z)_label; dlogits = (p - onehot) / B.
__global__ void k_softmax_ce(const float* __restrict__ logits, const int32_t* __restrict__ labels,
                             int B, int N, float* probs, bf16* dlogits, float* loss_rows,
                             int* status) {
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* z = logits + 1LL * b * N;
  const int tid = threadIdx.x, nw = blockDim.x >> 5;
  float m = -INFINITY;
  for (int j = tid; j < N; j += blockDim.x) m = fmaxf(m, z[j]);
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  if (tid < 32) {
    float v = tid < nw ? red[tid] : -INFINITY;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (tid == 0) red[0] = v;
  }
  __syncthreads();
  m = red[0];
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < N; j += blockDim.x) sum += expf(z[j] - m);
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((tid & 31) == 0) red[tid >> 5] = sum;
  __syncthreads();
  if (tid < 32) {
    float v = tid < nw ? red[tid] : 0.f;
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (tid == 0) red[0] = v;
  }
  __syncthreads();
  sum = red[0];
  int y = -1;
  if (labels) {
    y = labels[b];
    if (y < 0 || y >= N) {
      if (tid == 0) atomicOr(status, STATUS_LABEL_RANGE);
      y = -1;
    }
  }
  const float inv = 1.f / sum;
  const float invB = 1.f / static_cast<float>(B);
  for (int j = tid; j < N; j += blockDim.x) {
    const float p = expf(z[j] - m) * inv;
    if (probs) probs[1LL * b * N + j] = p;
    if (dlogits) dlogits[1LL * b * N + j] = __float2bfloat16_rn((p - (j == y ? 1.f : 0.f)) * invB);
  }
  if (tid == 0 && loss_rows) loss_rows[b] = y >= 0 ? -((z[y] - m) - logf(sum)) : 0.f;
}

__global__ void k_loss_mean(const float* __restrict__ rows, int B, float* out1, float* out2) {
  __shared__ float red[256];
  float s = 0.f;
  for (int i = threadIdx.x; i < B; i += blockDim.x) s += rows[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const float v = red[0] / static_cast<float>(B);
    if (out1) *out1 = v;
    if (out2) *out2 = v;
  }
}

// ------------------------------------------------------------------ bias gradients
constexpr int kColsumRows = 32;  // minimum rows per chunk (more chunks: more loads in flight)
constexpr int kColsumMaxChunks = 512;

// Rows per chunk: at least kColsumRows, a multiple of it, and no more than
// kColsumMaxChunks chunks (the bias update sums the chunks).
__host__ __device__ inline long long colsum_rows(long long rows) {
  long long per = (rows + kColsumMaxChunks - 1) / kColsumMaxChunks;
  per = (per + kColsumRows - 1) / kColsumRows * kColsumRows;
  return per < kColsumRows ? kColsumRows : per;
}

// Column sums of a bf16 [rows, cols] matrix (cols % 8 == 0) over chunks of
// colsum_rows(rows) rows.  Block (chunk, column block) covers Gb groups of 8
// columns; thread (lane row rl, group cg) sums its 8 columns over rows
// r0 + rl, r0 + rl + R, ... (four loads in flight), then the R lane rows are
// added in order.  Fixed order throughout: the sums are reproducible.
__device__ __forceinline__ int colsum_gb(int G) { return G <= 64 ? G : 16; }

__global__ void __launch_bounds__(256) k_colsum_partial(const bf16* __restrict__ m,
                                                        long long rows, int cols,
                                                        float* __restrict__ partial) {
  __shared__ float red[2048];
  const int G = cols >> 3;
  const int Gb = colsum_gb(G);
  const int R = 256 / Gb;
  const int g0 = blockIdx.y * Gb;
  const int gn = min(Gb, G - g0);
  const long long per = colsum_rows(rows);
  const long long r0 = 1LL * blockIdx.x * per;
  const long long r1 = min(rows, r0 + per);
  const int t = threadIdx.x;
  const int cg = t % Gb, rl = t / Gb;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (rl < R && cg < gn) {
    const bf16* base = m + (g0 + cg) * 8;
    long long r = r0 + rl;
    for (; r + 3LL * R < r1; r += 4LL * R) {
      uint4 u[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = *reinterpret_cast<const uint4*>(base + (r + q * R) * cols);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float f[8];
        unpack8(u[q], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += f[i];
      }
    }
    for (; r < r1; r += R) {
      float f[8];
      unpack8(*reinterpret_cast<const uint4*>(base + r * cols), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
  }
  if (rl < R) {
#pragma unroll
    for (int i = 0; i < 8; ++i) red[rl * Gb * 8 + cg * 8 + i] = acc[i];
  }
  __syncthreads();
  for (int c = t; c < gn * 8; c += blockDim.x) {
    float v = 0.f;
    for (int q = 0; q < R; ++q) v += red[q * Gb * 8 + c];
    partial[1LL * blockIdx.x * cols + g0 * 8 + c] = v;
  }
}

// ------------------------------------------------------------------ SGD
// [S] 3.4 "Training Procedure Details", update rule; [W] listing TRAIN_STEP:
// v <- momentum v - wd lr w - lr g ; w <- w + v, for every parameter.
// (sgd_one, the per-parameter update, is in kernels.h)

struct ConvIdx {
  long long fwd, dg, part_inner;
  int g, co;
};

// canonical p = ((o*K + kh)*K + kw)*Cg + ci
__device__ __forceinline__ ConvIdx conv_index(const ConvMap& m, long long p64) {
  const uint32_t p = static_cast<uint32_t>(p64);
  const int ci = static_cast<int>(p % m.Cg);
  uint32_t t = p / m.Cg;
  const int kw = static_cast<int>(t % m.K);
  t /= m.K;
  const int kh = static_cast<int>(t % m.K);
  const int o = static_cast<int>(t / m.K);
  const int Og = m.Cout / m.groups;
  ConvIdx r;
  r.g = o / Og;
  r.co = o - r.g * Og;
  if (m.s2d) {
    const int kg = ((kh >> 2) * 3 + (kw >> 2)) * 64 + ((kh & 3) * 4 + (kw & 3)) * 3 + ci;
    r.fwd = 1LL * o * 576 + kg;
    r.part_inner = kg;
    r.dg = -1;
  } else {
    r.part_inner = (1LL * kh * m.K + kw) * m.P + ci;
    r.fwd = 1LL * o * m.K * m.K * m.P + r.part_inner;
    r.dg = (((1LL * r.g * m.Cg + ci) * m.K + (m.K - 1 - kh)) * m.K + (m.K - 1 - kw)) * Og + r.co;
  }
  return r;
}

__global__ void k_sgd_conv(float* __restrict__ w, float* __restrict__ v,
                           const float* __restrict__ part, int S, ConvMap m, bf16* fwd, bf16* dg,
                           float* grads_out, const HParams* __restrict__ hpp) {
  const HParams hp = *hpp;
  const long long n = 1LL * m.Cout * m.K * m.K * m.Cg;
  const int Og = m.Cout / m.groups;
  const long long Kg = m.s2d ? 576 : 1LL * m.K * m.K * m.P;
  const long long split_stride = 1LL * m.groups * Og * Kg;
  for (long long p = blockIdx.x * 1LL * blockDim.x + threadIdx.x; p < n;
       p += 1LL * gridDim.x * blockDim.x) {
    const ConvIdx ix = conv_index(m, p);
    const long long base = (1LL * ix.g * Og + ix.co) * Kg + ix.part_inner;
    // the slices summed in order s = 0, 1, ...; loads issued four at a time
    float g = 0.f;
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) q[i] = part[(s + i) * split_stride + base];
#pragma unroll
      for (int i = 0; i < 4; ++i) g += q[i];
    }
    for (; s < S; ++s) g += part[s * split_stride + base];
    if (hp.update) {
      float wv = w[p], vv = v[p];
      sgd_one(wv, vv, g, hp);
      w[p] = wv;
      v[p] = vv;
      const bf16 hb = __float2bfloat16_rn(wv);
      fwd[ix.fwd] = hb;
      if (dg) dg[ix.dg] = hb;
    }
    if (grads_out) grads_out[p] = g;
  }
}

// k_sgd_conv for four consecutive parameters per thread (same kernel tap,
// four consecutive input channels: Cg % 4 == 0, not the space-to-depth
// form, no flipped copy), so that every partial-sum, weight and momentum
// access is a 16-byte vector and four splits' loads are in flight at once.
// Same summation order (slices s = 0, 1, ...) and update as k_sgd_conv.
__global__ void k_sgd_conv4(float* __restrict__ w, float* __restrict__ v,
                            const float* __restrict__ part, int S, ConvMap m, bf16* fwd,
                            float* grads_out, const HParams* __restrict__ hpp) {
  const HParams hp = *hpp;
  const long long n4 = 1LL * m.Cout * m.K * m.K * m.Cg / 4;
  const int Og = m.Cout / m.groups;
  const long long Kg = 1LL * m.K * m.K * m.P;
  const long long split4 = 1LL * m.groups * Og * Kg / 4;  // split stride in float4
  const float4* part4 = reinterpret_cast<const float4*>(part);
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n4;
       q += 1LL * gridDim.x * blockDim.x) {
    const ConvIdx ix = conv_index(m, 4 * q);
    const long long base4 = ((1LL * ix.g * Og + ix.co) * Kg + ix.part_inner) / 4;
    float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float4 t[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) t[i] = part4[(s + i) * split4 + base4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        g.x += t[i].x;
        g.y += t[i].y;
        g.z += t[i].z;
        g.w += t[i].w;
      }
    }
    for (; s < S; ++s) {
      const float4 t = part4[s * split4 + base4];
      g.x += t.x;
      g.y += t.y;
      g.z += t.z;
      g.w += t.w;
    }
    if (hp.update) {
      float4 wv = reinterpret_cast<float4*>(w)[q];
      float4 vv = reinterpret_cast<float4*>(v)[q];
      sgd_one(wv.x, vv.x, g.x, hp);
      sgd_one(wv.y, vv.y, g.y, hp);
      sgd_one(wv.z, vv.z, g.z, hp);
      sgd_one(wv.w, vv.w, g.w, hp);
      reinterpret_cast<float4*>(w)[q] = wv;
      reinterpret_cast<float4*>(v)[q] = vv;
      uint2 u;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(wv.x, wv.y);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(wv.z, wv.w);
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(fwd + ix.fwd) = u;
    }
    if (grads_out) reinterpret_cast<float4*>(grads_out)[q] = g;
  }
}

__global__ void k_conv_shadows(const float* __restrict__ w, ConvMap m, bf16* fwd, bf16* dg) {
  const long long n = 1LL * m.Cout * m.K * m.K * m.Cg;
  for (long long p = blockIdx.x * 1LL * blockDim.x + threadIdx.x; p < n;
       p += 1LL * gridDim.x * blockDim.x) {
    const ConvIdx ix = conv_index(m, p);
    const bf16 hb = __float2bfloat16_rn(w[p]);
    fwd[ix.fwd] = hb;
    if (dg) dg[ix.dg] = hb;
  }
}

__global__ void k_sgd_dense(float* __restrict__ w, float* __restrict__ v,
                            const float* __restrict__ g, long long n, bf16* shadow,
                            float* grads_out, const HParams* __restrict__ hpp) {
  const HParams hp = *hpp;
  const long long n4 = n / 4;
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n4;
       q += 1LL * gridDim.x * blockDim.x) {
    const float4 gv = reinterpret_cast<const float4*>(g)[q];
    if (grads_out) reinterpret_cast<float4*>(grads_out)[q] = gv;
    if (!hp.update) continue;
    float4 wv = reinterpret_cast<float4*>(w)[q];
    float4 vv = reinterpret_cast<float4*>(v)[q];
    sgd_one(wv.x, vv.x, gv.x, hp);
    sgd_one(wv.y, vv.y, gv.y, hp);
    sgd_one(wv.z, vv.z, gv.z, hp);
    sgd_one(wv.w, vv.w, gv.w, hp);
    reinterpret_cast<float4*>(w)[q] = wv;
    reinterpret_cast<float4*>(v)[q] = vv;
    if (shadow) {
      uint2 u;
      __nv_bfloat162 h0 = __floats2bfloat162_rn(wv.x, wv.y);
      __nv_bfloat162 h1 = __floats2bfloat162_rn(wv.z, wv.w);
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      reinterpret_cast<uint2*>(shadow)[q] = u;
    }
  }
}

// One block per 32 channels: thread (tx, ty) sums the rows ty, ty + 32, ...
// of channel tx (four loads in flight), then row ty = 0 adds the 32
// row-group sums in order and applies the update.  The rows are fp32
// partial column sums (T = float), or, for a short matrix, the bf16
// gradient rows themselves (T = bf16: the column sum is the bias gradient).
template <typename T>
__device__ __forceinline__ void bias_block(float* __restrict__ b, float* __restrict__ v,
                                           const T* __restrict__ partial, int chunks, int n,
                                           float* grads_out, const HParams* __restrict__ hpp,
                                           int blk, float (&red)[32][33]) {
  const int tx = threadIdx.x, ty = threadIdx.y;
  const int i = blk * 32 + tx;
  float g = 0.f;
  if (i < n) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const T* p = partial + i;
    const size_t n32 = static_cast<size_t>(n) * 32;
    int c = ty;
    for (; c + 96 < chunks; c += 128) {
      const T* q = p + static_cast<size_t>(c) * n;
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] += static_cast<float>(q[u * n32]);
    }
    for (; c < chunks; c += 32) acc[0] += static_cast<float>(p[static_cast<size_t>(c) * n]);
    g = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
  red[ty][tx] = g;
  __syncthreads();
  if (ty == 0 && i < n) {
    float sum = 0.f;
#pragma unroll 8
    for (int q = 0; q < 32; ++q) sum += red[q][tx];
    const HParams hp = *hpp;
    if (hp.update) {
      float wv = b[i], vv = v[i];
      sgd_one(wv, vv, sum, hp);
      b[i] = wv;
      v[i] = vv;
    }
    if (grads_out) grads_out[i] = sum;
  }
}

template <typename T>
__global__ void __launch_bounds__(1024) k_sgd_bias(float* __restrict__ b, float* __restrict__ v,
                                                   const T* __restrict__ partial, int chunks,
                                                   int n, float* grads_out,
                                                   const HParams* __restrict__ hpp) {
  __shared__ float red[32][33];
  bias_block<T>(b, v, partial, chunks, n, grads_out, hpp, blockIdx.x, red);
}

// Several layers' bias updates in one launch: block k belongs to the last
// job whose first block is <= k.
__global__ void __launch_bounds__(1024) k_sgd_bias_jobs(BiasJobs jobs,
                                                        const HParams* __restrict__ hpp) {
  __shared__ float red[32][33];
  int k = 0;
  while (k + 1 < jobs.count && static_cast<int>(blockIdx.x) >= jobs.j[k + 1].block0) ++k;
  const BiasJob& J = jobs.j[k];
  bias_block<float>(J.b, J.v, J.partial, J.chunks, J.n, J.grads_out, hpp,
                    static_cast<int>(blockIdx.x) - J.block0, red);
}

// [S] 3.4 "Training Procedure Details", update rule, on a range of the
// parameter blob with a gradient that arrives scaled: g = scale * gsum (the
// sum of the ranks' gradients of their own batch means, scale = 1 / ranks).
__global__ void k_sgd_range(float* __restrict__ w, float* __restrict__ v,
                            const float* __restrict__ gsum, long long n, float scale, float lr,
                            float momentum, float wd) {
  for (long long p = blockIdx.x * 1LL * blockDim.x + threadIdx.x; p < n;
       p += 1LL * gridDim.x * blockDim.x) {
    const float g = scale * gsum[p];
    const float vn = momentum * v[p] - wd * lr * w[p] - lr * g;
    v[p] = vn;
    w[p] += vn;
  }
}

__global__ void k_f32_to_bf16(const float* __restrict__ w, bf16* __restrict__ out, long long n) {
  for (long long i = blockIdx.x * 1LL * blockDim.x + threadIdx.x; i < n;
       i += 1LL * gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(w[i]);
}

__global__ void k_f32_from_bf16(const bf16* __restrict__ in, float* __restrict__ out, long long n) {
  for (long long i = blockIdx.x * 1LL * blockDim.x + threadIdx.x; i < n;
       i += 1LL * gridDim.x * blockDim.x)
    out[i] = __bfloat162float(in[i]);
}

// ------------------------------------------------------------------ init
// [S] 3.4 "Training Procedure Details", weight initialisation: zero-mean
// Gaussian with standard deviation 0.01.  Normals from Box-Muller on Philox
// words: Philox((q, tag, 0xC0, 0), seed) gives elements 4q .. 4q+3.
__global__ void k_init_normal(float* __restrict__ w, long long n, float stdv, uint32_t k0,
                              uint32_t k1, uint32_t tag) {
  const long long n4 = (n + 3) / 4;
  for (long long q = blockIdx.x * 1LL * blockDim.x + threadIdx.x; q < n4;
       q += 1LL * gridDim.x * blockDim.x) {
    const U4 r = philox4x32_10(U4{static_cast<uint32_t>(q), tag, 0xC0u, 0u}, k0, k1);
    const float r1 = sqrtf(-2.f * logf(word_unit(r.x)));
    const float r2 = sqrtf(-2.f * logf(word_unit(r.z)));
    float s1, c1, s2, c2;
    sincospif(2.f * word_unit(r.y), &s1, &c1);
    sincospif(2.f * word_unit(r.w), &s2, &c2);
    const float z[4] = {r1 * c1, r1 * s1, r2 * c2, r2 * s2};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (q * 4 + i < n) w[q * 4 + i] = stdv * z[i];
  }
}

__global__ void k_fill(float* __restrict__ w, long long n, float value) {
  for (long long i = blockIdx.x * 1LL * blockDim.x + threadIdx.x; i < n;
       i += 1LL * gridDim.x * blockDim.x)
    w[i] = value;
}

// ------------------------------------------------------------------ augmentation
// [S] 3.4 "Data Augmentation": Form 1, a 224x224 patch at offset (oy, ox) in
// 0..31 with an optional horizontal reflection; Form 2, the same colour
// offset [p1 p2 p3][a1 l1, a2 l2, a3 l3]^T added to every pixel of the image,
// a_i ~ N(0, 0.1^2).  Per-pixel mean subtracted first ([S] 3.2).  Draws for
// image i at step t: word 0 of Philox((i, 0xA0, t, 0)) -> bits 0-4 oy,
// bits 5-9 ox, bit 10 reflection; Philox((i, 0xA1, t, 0)) -> Box-Muller
// pairs (words 0, 1 -> a1, a2; words 2, 3 -> a3 from the cosine branch).
struct AugDraw {
  int oy, ox, flip;
  float add[3];
};

__device__ __forceinline__ AugDraw aug_draw(const HParams& hp, uint32_t img, const float* pv,
                                            const float* pl) {
  AugDraw d;
  const U4 r0 = philox4x32_10(U4{img, 0xA0u, hp.step, 0u}, hp.seed_lo, hp.seed_hi);
  d.oy = static_cast<int>(r0.x & 31u);
  d.ox = static_cast<int>((r0.x >> 5) & 31u);
  d.flip = static_cast<int>((r0.x >> 10) & 1u);
  const U4 r1 = philox4x32_10(U4{img, 0xA1u, hp.step, 0u}, hp.seed_lo, hp.seed_hi);
  const float m1 = sqrtf(-2.f * logf(word_unit(r1.x)));
  const float m2 = sqrtf(-2.f * logf(word_unit(r1.z)));
  float s1, c1, s2, c2;
  sincospif(2.f * word_unit(r1.y), &s1, &c1);
  sincospif(2.f * word_unit(r1.w), &s2, &c2);
  const float a[3] = {0.1f * m1 * c1, 0.1f * m1 * s1, 0.1f * m2 * c2};
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 3; ++i) s += pv[c * 3 + i] * (a[i] * pl[i]);
    d.add[c] = s;
  }
  return d;
}

// One block per (image, run of kAugRows output rows): the image's draw
// (Philox + Box-Muller, one thread) is taken once per run, not once per row,
// and the run's rows are written element by element (bf16, coalesced).
constexpr int kAugRows = 8;
__global__ void k_augment(const uint8_t* __restrict__ src, int B, const float* __restrict__ mean,
                          const float* __restrict__ pca_vec, const float* __restrict__ pca_val,
                          const HParams* __restrict__ hpp, bf16* __restrict__ out) {
  const HParams hp = *hpp;
  __shared__ AugDraw d;
  __shared__ float pv[9], pl[3];
  if (threadIdx.x < 9) pv[threadIdx.x] = pca_vec[threadIdx.x];
  if (threadIdx.x < 3) pl[threadIdx.x] = pca_val[threadIdx.x];
  constexpr int kRuns = (227 + kAugRows - 1) / kAugRows;
  for (long long job = blockIdx.x; job < 1LL * B * kRuns; job += gridDim.x) {
    const int b = static_cast<int>(job / kRuns);
    const int y0 = static_cast<int>(job % kRuns) * kAugRows;
    const int rows = min(kAugRows, 227 - y0);
    __syncthreads();  // pv / pl written; the previous run's d no longer read
    if (threadIdx.x == 0) d = aug_draw(hp, static_cast<uint32_t>(b), pv, pl);
    __syncthreads();
    const uint8_t* simg = src + 1LL * b * 256 * 256 * 3;
    bf16* orun = out + (1LL * b * 227 + y0) * 227 * 3;
    for (int e = threadIdx.x; e < rows * 227 * 3; e += blockDim.x) {
      const int r = e / (227 * 3);
      const int q = e - r * (227 * 3);
      const int x = q / 3, c = q - x * 3;
      const int y = y0 + r;
      float v = 0.f;
      if (y < 224 && x < 224) {
        const int sy = d.oy + y;
        const int sx = d.flip ? d.ox + 223 - x : d.ox + x;
        const int si = (sy * 256 + sx) * 3 + c;
        v = static_cast<float>(simg[si]) - mean[si] + d.add[c];
      }
      orun[e] = __float2bfloat16_rn(v);
    }
  }
}

// [S] 3.4 "Data Augmentation", test time: four corner patches and the centre
// patch, then their reflections (order TL, TR, BL, BR, centre, reflected x5).
__constant__ int kTenOy[5] = {0, 0, 32, 32, 16};
__constant__ int kTenOx[5] = {0, 32, 0, 32, 16};

__global__ void k_tencrop_inputs(const uint8_t* __restrict__ src, int B,
                                 const float* __restrict__ mean, bf16* __restrict__ out) {
  for (long long job = blockIdx.x; job < 1LL * B * 10 * 227; job += gridDim.x) {
    const int img = static_cast<int>(job / 227);
    const int y = static_cast<int>(job % 227);
    const int b = img / 10, p = img % 10;
    const int oy = kTenOy[p % 5], ox = kTenOx[p % 5], flip = p >= 5;
    bf16* orow = out + (1LL * img * 227 + y) * 227 * 3;
    for (int e = threadIdx.x; e < 227 * 3; e += blockDim.x) {
      const int x = e / 3, c = e - x * 3;
      float v = 0.f;
      if (y < 224 && x < 224) {
        const int sy = oy + y;
        const int sx = flip ? ox + 223 - x : ox + x;
        const long long si = (1LL * sy * 256 + sx) * 3 + c;
        v = static_cast<float>(src[1LL * b * 256 * 256 * 3 + si]) - mean[si];
      }
      orow[e] = __float2bfloat16_rn(v);
    }
  }
}

// Average of the ten softmax outputs, then top-5 by descending probability,
// ties to the lower class index.
// Mean of n probability rows per image, then its top 5 (descending, ties
// to the lower class).  Row m of image b starts at probs + m * stride_m +
// b * stride_b; the n rows are added in order m = 0, 1, ... and divided by n.
// Ten-crop: the 10 crops of an image are consecutive rows; ensemble: model
// m's rows form the m-th [B][N] block.
__global__ void k_avg_top5(const float* __restrict__ probs, int n, long long stride_m,
                           long long stride_b, int N, float* __restrict__ avg,
                           int32_t* __restrict__ top5) {
  extern __shared__ float sp[];
  __shared__ float bv[32];
  __shared__ int bi[32];
  const int b = blockIdx.x;
  for (int j = threadIdx.x; j < N; j += blockDim.x) {
    float s = 0.f;
    for (int p = 0; p < n; ++p) s += probs[p * stride_m + b * stride_b + j];
    s = s / static_cast<float>(n);
    sp[j] = s;
    avg[1LL * b * N + j] = s;
  }
  __syncthreads();
  const int nw = blockDim.x >> 5;
  for (int k = 0; k < 5; ++k) {
    float best = -INFINITY;
    int idx = 0x7fffffff;
    for (int j = threadIdx.x; j < N; j += blockDim.x) {
      const float v = sp[j];
      if (v > best || (v == best && j < idx)) {
        best = v;
        idx = j;
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, idx, o);
      if (ov > best || (ov == best && oi < idx)) {
        best = ov;
        idx = oi;
      }
    }
    if ((threadIdx.x & 31) == 0) {
      bv[threadIdx.x >> 5] = best;
      bi[threadIdx.x >> 5] = idx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float b0 = bv[0];
      int i0 = bi[0];
      for (int w = 1; w < nw; ++w)
        if (bv[w] > b0 || (bv[w] == b0 && bi[w] < i0)) {
          b0 = bv[w];
          i0 = bi[w];
        }
      top5[b * 5 + k] = i0;
      sp[i0] = -INFINITY;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ fp32 path
// wt[g][t][co] with t = (kh*K + kw)*Cg + ci, co within the group.
__global__ void k_conv_wt_f32(const float* __restrict__ w, float* __restrict__ wt, int Cout, int K,
                              int Cg, int groups) {
  const long long n = 1LL * Cout * K * K * Cg;
  const int Og = Cout / groups;
  const long long T = 1LL * K * K * Cg;
  for (long long p = blockIdx.x * 1LL * blockDim.x + threadIdx.x; p < n;
       p += 1LL * gridDim.x * blockDim.x) {
    const long long t = p % T;
    const int o = static_cast<int>(p / T);
    const int g = o / Og, co = o - g * Og;
    wt[(1LL * g * T + t) * Og + co] = w[p];
  }
}

__global__ void k_conv_fwd_f32(const float* __restrict__ x, const float* __restrict__ wt,
                               const float* __restrict__ bias, float* __restrict__ y, int B, int H,
                               int W, int Cin, int Cout, int K, int stride, int pad, int groups,
                               int Ho, int Wo) {
  const int Og = Cout / groups, Cg = Cin / groups;
  const int g = blockIdx.z;
  const int co = blockIdx.y * blockDim.x + threadIdx.x;
  const long long T = 1LL * K * K * Cg;
  for (long long pix = blockIdx.x; pix < 1LL * B * Ho * Wo; pix += gridDim.x) {
    if (co >= Og) continue;
    const int ow = static_cast<int>(pix % Wo);
    const int oh = static_cast<int>((pix / Wo) % Ho);
    const int b = static_cast<int>(pix / (1LL * Wo * Ho));
    float acc = bias[g * Og + co];
    for (int kh = 0; kh < K; ++kh) {
      const int ih = oh * stride - pad + kh;
      if (ih < 0 || ih >= H) continue;
      for (int kw = 0; kw < K; ++kw) {
        const int iw = ow * stride - pad + kw;
        if (iw < 0 || iw >= W) continue;
        const float* xp = x + ((1LL * b * H + ih) * W + iw) * Cin + g * Cg;
        const float* wp = wt + (1LL * g * T + (1LL * kh * K + kw) * Cg) * Og + co;
        for (int ci = 0; ci < Cg; ++ci) acc = fmaf(__ldg(xp + ci), wp[1LL * ci * Og], acc);
      }
    }
    y[pix * Cout + g * Og + co] = acc > 0.f ? acc : 0.f;
  }
}

// Register-tiled fp32 direct convolution (+ bias + ReLU) for small batches.
// A block computes kTileP consecutive output pixels of one output row for 32
// output channels of one group (lane = channel, kTileP accumulators).  The
// input patch the tile reads (K rows x ((kTileP - 1) * stride + K) columns x
// Cg channels, zero outside the map) is staged in shared memory, so every
// weight loaded from global memory serves kTileP pixels.  The block's
// kConvWarps warps split the reduction (SPLIT_CI: each takes an equal share
// of the input channels of every tap, Cg % (4 * kConvWarps) == 0; else a
// share of the taps) and their sums are added in warp order.
constexpr int kTileP = 8;
constexpr int kConvWarps = 8;
template <bool SPLIT_CI>
__global__ void __launch_bounds__(32 * kConvWarps) k_conv_fwd_f32_tiled(
    const float* __restrict__ x, const float* __restrict__ wt, const float* __restrict__ bias,
    float* __restrict__ y, int H, int W, int Cin, int Cout, int K, int stride, int pad,
    int groups, int Ho, int Wo) {
  extern __shared__ float4 xs4[];
  float* xs = reinterpret_cast<float*>(xs4);
  const int Og = Cout / groups, Cg = Cin / groups;
  const int g = blockIdx.z;
  const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
  const int co = blockIdx.y * 32 + lane;
  const int tiles_w = (Wo + kTileP - 1) / kTileP;
  const int ow0 = (blockIdx.x % tiles_w) * kTileP;
  const int oh = (blockIdx.x / tiles_w) % Ho;
  const int b = blockIdx.x / (tiles_w * Ho);
  const int PW = (kTileP - 1) * stride + K;  // patch columns
  const int ih0 = oh * stride - pad, iw0 = ow0 * stride - pad;
  const int n = K * PW * Cg;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int ci = i % Cg;
    const int col = (i / Cg) % PW;
    const int r = i / (Cg * PW);
    const int ih = ih0 + r, iw = iw0 + col;
    xs[i] = (ih >= 0 && ih < H && iw >= 0 && iw < W)
                ? x[((static_cast<size_t>(b) * H + ih) * W + iw) * Cin + g * Cg + ci]
                : 0.f;
  }
  __syncthreads();
  float acc[kTileP];
#pragma unroll
  for (int p = 0; p < kTileP; ++p) acc[p] = 0.f;
  if (co < Og) {
    const float* wg = wt + static_cast<size_t>(g) * K * K * Cg * Og + co;
    const int taps = K * K;
    const int t0 = SPLIT_CI ? 0 : wq * taps / kConvWarps;
    const int t1 = SPLIT_CI ? taps : (wq + 1) * taps / kConvWarps;
    const int c0 = SPLIT_CI ? wq * (Cg / kConvWarps) : 0;
    const int c1 = SPLIT_CI ? c0 + Cg / kConvWarps : Cg;
    for (int t = t0; t < t1; ++t) {
      const int kh = t / K, kw = t - kh * K;
      const float* wp = wg + static_cast<size_t>(t) * Cg * Og;
      const float* xr = xs + (kh * PW + kw) * Cg;
      if (SPLIT_CI) {
#pragma unroll 2
        for (int ci = c0; ci < c1; ci += 4) {
          const float w0 = wp[(ci + 0) * Og], w1 = wp[(ci + 1) * Og];
          const float w2 = wp[(ci + 2) * Og], w3 = wp[(ci + 3) * Og];
#pragma unroll
          for (int p = 0; p < kTileP; ++p) {
            const float4 v = *reinterpret_cast<const float4*>(xr + p * stride * Cg + ci);
            acc[p] = fmaf(v.x, w0, acc[p]);
            acc[p] = fmaf(v.y, w1, acc[p]);
            acc[p] = fmaf(v.z, w2, acc[p]);
            acc[p] = fmaf(v.w, w3, acc[p]);
          }
        }
      } else {
        for (int ci = c0; ci < c1; ++ci) {
          const float w0 = wp[ci * Og];
#pragma unroll
          for (int p = 0; p < kTileP; ++p) acc[p] = fmaf(xr[p * stride * Cg + ci], w0, acc[p]);
        }
      }
    }
  }
  __syncthreads();  // the patch is no longer read: its space takes the warp sums
  float* red = xs;  // [warp][pixel][lane]
#pragma unroll
  for (int p = 0; p < kTileP; ++p) red[(wq * kTileP + p) * 32 + lane] = acc[p];
  __syncthreads();
  if (wq != 0 || co >= Og) return;
  const float bv = bias[g * Og + co];
#pragma unroll
  for (int p = 0; p < kTileP; ++p) {
    const int ow = ow0 + p;
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < kConvWarps; ++q) v += red[(q * kTileP + p) * 32 + lane];
    v += bv;
    if (ow < Wo)
      y[((static_cast<size_t>(b) * Ho + oh) * Wo + ow) * Cout + g * Og + co] = v > 0.f ? v : 0.f;
  }
}

// fp32 FC row dot products with 16-byte loads, four in flight per lane
// (In % 4 == 0, rows 16-byte aligned).
__global__ void k_fc_fwd_f32_v4(const float* __restrict__ x, const float* __restrict__ w,
                                const float* __restrict__ bias, float* __restrict__ y, int B,
                                int In, int Out, int relu, float scale) {
  const int lane = threadIdx.x & 31;
  const long long warps = 1LL * gridDim.x * (blockDim.x >> 5);
  const int n4 = In >> 2;
  for (long long job = blockIdx.x * 1LL * (blockDim.x >> 5) + (threadIdx.x >> 5);
       job < 1LL * B * Out; job += warps) {
    const int b = static_cast<int>(job / Out), o = static_cast<int>(job % Out);
    const float4* xr = reinterpret_cast<const float4*>(x + 1LL * b * In);
    const float4* wr = reinterpret_cast<const float4*>(w + 1LL * o * In);
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int i = lane;
    for (; i + 96 < n4; i += 128) {
      float4 wv[4], xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        wv[u] = wr[i + 32 * u];
        xv[u] = xr[i + 32 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        s0 = fmaf(xv[u].x, wv[u].x, s0);
        s1 = fmaf(xv[u].y, wv[u].y, s1);
        s2 = fmaf(xv[u].z, wv[u].z, s2);
        s3 = fmaf(xv[u].w, wv[u].w, s3);
      }
    }
    for (; i < n4; i += 32) {
      const float4 wv = wr[i], xv = xr[i];
      s0 = fmaf(xv.x, wv.x, s0);
      s1 = fmaf(xv.y, wv.y, s1);
      s2 = fmaf(xv.z, wv.z, s2);
      s3 = fmaf(xv.w, wv.w, s3);
    }
    float s = (s0 + s1) + (s2 + s3);
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      float v = s + bias[o];
      if (relu) v = v > 0.f ? v : 0.f;
      y[job] = v * scale;
    }
  }
}

__global__ void k_fc_fwd_f32(const float* __restrict__ x, const float* __restrict__ w,
                             const float* __restrict__ bias, float* __restrict__ y, int B, int In,
                             int Out, int relu, float scale) {
  const int lane = threadIdx.x & 31;
  const long long warps = 1LL * gridDim.x * (blockDim.x >> 5);
  for (long long job = blockIdx.x * 1LL * (blockDim.x >> 5) + (threadIdx.x >> 5);
       job < 1LL * B * Out; job += warps) {
    const int b = static_cast<int>(job / Out), o = static_cast<int>(job % Out);
    const float* xr = x + 1LL * b * In;
    const float* wr = w + 1LL * o * In;
    float s = 0.f;
    for (int i = lane; i < In; i += 32) s = fmaf(xr[i], wr[i], s);
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) {
      float v = s + bias[o];
      if (relu) v = v > 0.f ? v : 0.f;
      y[job] = v * scale;
    }
  }
}

}  // namespace

// The bounded wait of the pipelined kernels, made to run out: one thread
// waits on an mbarrier that nothing arrives at, with a limit of `limit`
// clocks; on expiry the wait records TIMEOUT in *status and returns, and so
// does the kernel.
__global__ void k_wait_probe(int* status, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait_limit(b, 0, status, &abort_flag, limit);
}

// ================================================================== launchers
namespace {
std::atomic<int64_t> g_launches{0};
}
int64_t launch_counter() { return g_launches.load(); }
void count_launch() { g_launches.fetch_add(1); }
void count_launch_n(int64_t n) { g_launches.fetch_add(n); }

void launch_wait_probe(int* status, long long limit_cycles, cudaStream_t s) {
  k_wait_probe<<<1, 32, 0, s>>>(status, limit_cycles);
  count_launch();
}
void launch_write_hparams(HParams* hp, HParams v, cudaStream_t s) {
  k_write_hparams<<<1, 1, 0, s>>>(hp, v);
  count_launch();
}

void launch_s2d(const bf16* x, bf16* xs, int B, cudaStream_t s) {
  k_s2d<<<B * ((57 + kS2dRows - 1) / kS2dRows), 256, 0, s>>>(x, xs, B);
  count_launch();
}
void launch_lrn_fwd(const bf16* a, bf16* b, long long P, int C, int, float k, float alpha,
                    float beta, cudaStream_t s) {
  if (beta == 0.75f)
    k_lrn_fwd<true><<<grid_for(P * (C / 8), 256), 256, 0, s>>>(a, b, P, C, k, alpha, beta);
  else
    k_lrn_fwd<false><<<grid_for(P * (C / 8), 256), 256, 0, s>>>(a, b, P, C, k, alpha, beta);
  count_launch();
}
void launch_lrn_bwd(const bf16* a, const bf16* g, bf16* da, long long P, int C, int, float k,
                    float alpha, float beta, cudaStream_t s) {
  if (beta == 0.75f)
    k_lrn_bwd<true><<<grid_for(P * (C / 8), 256), 256, 0, s>>>(a, g, da, P, C, k, alpha, beta);
  else
    k_lrn_bwd<false><<<grid_for(P * (C / 8), 256), 256, 0, s>>>(a, g, da, P, C, k, alpha, beta);
  count_launch();
}
void launch_lrn_fwd_f32(const float* a, float* b, long long P, int C, int, float k, float alpha,
                        float beta, cudaStream_t s) {
  k_lrn_fwd_f32<<<grid_for(P * C, 256), 256, 0, s>>>(a, b, P, C, k, alpha, beta);
  count_launch();
}
void launch_pool_fwd(const bf16* x, bf16* y, uint8_t* am, int B, int H, int W, int C, int z,
                     int st, cudaStream_t s) {
  const int Ho = (H - z) / st + 1, Wo = (W - z) / st + 1;
  const int grid = grid_for(1LL * B * Ho * Wo * (C / 8), 256);
  if (z == 3)
    k_pool_fwd<3><<<grid, 256, 0, s>>>(x, y, am, B, H, W, C, st);
  else
    k_pool_fwd<2><<<grid, 256, 0, s>>>(x, y, am, B, H, W, C, st);
  count_launch();
}
constexpr int kPoolBwdPartBlocks = 148 * 8;  // grid when the bias sums are produced
int pool_bwd_parts(int B, int H, int W, int C) {
  if (C < 8 || C % 8 || 256 % (C / 8)) return 0;
  const int g = grid_for(1LL * B * H * W * (C / 8), 256);
  return g < kPoolBwdPartBlocks ? g : kPoolBwdPartBlocks;
}
int launch_pool_bwd(const bf16* dy, const uint8_t* am, const bf16* pooled, bf16* dx, int B,
                    int H, int W, int C, int z, int st, int relu_mask, cudaStream_t s,
                    float* bias_part) {
  const int parts = bias_part ? pool_bwd_parts(B, H, W, C) : 0;
  const int grid = parts > 0 ? parts : grid_for(1LL * B * H * W * (C / 8), 256);
  k_pool_bwd<<<grid, 256, 0, s>>>(dy, am, pooled, dx, B, H, W, C, z, st, relu_mask,
                                  parts > 0 ? bias_part : nullptr);
  count_launch();
  return parts;
}
bool launch_lrn_pool_fwd(const bf16* a, bf16* lo, bf16* y, uint8_t* am, int B, int H, int W,
                         int C, int z, float k, float alpha, float beta, cudaStream_t s) {
  if (C % kSlab || (z != 2 && z != 3) || H < z || W < z) return false;
  const int Ho = (H - z) / 2 + 1;
  // rows a tile normalises: 2T - 2 + z for an inner tile; the last tile also
  // takes the rows below its last window, at most 2T + 2 in all
  const int rows = 2 * kPoolTileRows + 2;
  const size_t smem = static_cast<size_t>(rows) * W * kSlab * 2;
  if (smem > 48 * 1024) return false;
  const dim3 grid(C / kSlab, (Ho + kPoolTileRows - 1) / kPoolTileRows, B);
  auto go = [&](auto kern) { kern<<<grid, 256, smem, s>>>(a, lo, y, am, H, W, C, k, alpha, beta); };
  const bool b34 = beta == 0.75f;
  if (z == 3 && H == 55 && W == 55)
    b34 ? go(k_lrn_pool_fwd<3, 55, true>) : go(k_lrn_pool_fwd<3, 55, false>);
  else if (z == 3 && H == 27 && W == 27)
    b34 ? go(k_lrn_pool_fwd<3, 27, true>) : go(k_lrn_pool_fwd<3, 27, false>);
  else if (z == 3)
    b34 ? go(k_lrn_pool_fwd<3, 0, true>) : go(k_lrn_pool_fwd<3, 0, false>);
  else
    b34 ? go(k_lrn_pool_fwd<2, 0, true>) : go(k_lrn_pool_fwd<2, 0, false>);
  count_launch();
  return true;
}
__device__ int g_aux_status;
int* aux_status_word() {
  void* p = nullptr;
  return cudaGetSymbolAddress(&p, g_aux_status) == cudaSuccess ? static_cast<int*>(p) : nullptr;
}
constexpr int kPoolLrnBlocks = 148 * 8;  // persistent blocks: eight per SM
// quads of 2 x 2 pixels per block (one 8-channel unit per thread)
inline int pool_lrn_quads_per_block(int C) { return 256 / (C / 8); }
// quads per block of the warp-segment kernel (8 warps of 32 / (C / 8) quads)
inline int pool_lrn_quads_per_block_w(int C) { return 8 * (32 / (C / 8)); }
inline bool pool_lrn_use_warp_kernel(int C) { return C >= 8 && C <= 256; }
// Launch shape of the staged kernel: stages per block, threads, dynamic
// shared memory and blocks (persistent, over the SMs).  False if the shape
// does not suit it (bulk copies need 16-byte rows; at most 448 threads).
struct PlbCfg {
  int nst, threads, smem, blocks;
};
bool pool_lrn_staged_cfg(int B, int H, int W, int C, int z, PlbCfg* c) {
  if (C <= 0 || C % 8 || (z != 2 && z != 3) || H < z || W < z) return false;
  const int Wo = (W - z) / 2 + 1;
  if ((W * C * 2) % 16 || (Wo * C) % 16) return false;
  const int QW = (W + 1) / 2, QH = (H + 1) / 2;
  const int threads = (QW * (C / 8) + 31) / 32 * 32;
  if (threads > 448) return false;
  const PlbGeom G = plb_geom(W, Wo, C);
  constexpr int kBudget = 227 * 1024, kSmPerSm = 228 * 1024;
  // registers per thread as allocated (the kernel is built for two blocks of
  // 448 threads per SM: at most 72)
  constexpr int kRegs = 72;
  // the most items in flight per SM (stages x resident blocks); ties go to
  // fewer stages and more blocks
  int best = 0;
  for (int nst = 2; nst <= 4; ++nst) {
    const int smem = nst * G.stage + 2 * threads * 16 + 8 * nst + 16;
    if (smem > kBudget) break;
    int bps = kSmPerSm / (smem + 1024);
    bps = std::min(bps, 2048 / threads);
    bps = std::min(bps, 65536 / (kRegs * threads));
    if (bps < 1) break;
    if (nst * bps > best) {
      best = nst * bps;
      c->nst = nst;
      c->smem = smem;
      c->blocks = bps;
    }
  }
  if (!best) return false;
  // the bias column sums reuse the first stage: QW x C floats
  if (QW * C * 4 > c->nst * G.stage) return false;
  c->threads = threads;
  const long long items = 1LL * B * QH;
  const long long grid = std::min<long long>(items, 148LL * c->blocks);
  c->blocks = static_cast<int>(grid);
  return true;
}
// Rows of bias partial sums the block-per-row kernels write.
static int pool_lrn_bwd_parts_unstaged(int B, int H, int W, int C) {
  if (C <= 0 || C % 8 || C > 2048) return 0;
  const long long nquads = 1LL * B * ((H + 1) / 2) * ((W + 1) / 2);
  const int nq = pool_lrn_use_warp_kernel(C) ? pool_lrn_quads_per_block_w(C)
                                             : pool_lrn_quads_per_block(C);
  const long long groups = nq > 0 ? (nquads + nq - 1) / nq : 0;
  return static_cast<int>(groups < kPoolLrnBlocks ? groups : kPoolLrnBlocks);
}
int pool_lrn_bwd_parts(int B, int H, int W, int C, int z) {
  PlbCfg pc;
  const int staged = pool_lrn_staged_cfg(B, H, W, C, z, &pc) ? pc.blocks : 0;
  return std::max(staged, pool_lrn_bwd_parts_unstaged(B, H, W, C));
}
int launch_pool_lrn_bwd(const bf16* dy, const uint8_t* am, const bf16* a, bf16* dl, bf16* da,
                        int B, int H, int W, int C, int z, float k, float alpha, float beta,
                        float* bias_part, int* status, cudaStream_t s) {
  if (C % kSlab || C > 2048 || (z != 2 && z != 3) || H < z || W < z) return 0;
  const long long npix = 1LL * B * H * W;
  if (npix * C >= (1LL << 31)) return 0;  // 32-bit element offsets
  const bool b34 = beta == 0.75f;
  const int blocks = pool_lrn_bwd_parts_unstaged(B, H, W, C);
  const int nq = pool_lrn_quads_per_block(C);
  if (nq < 1 || blocks < 1) return 0;
  const int nquads = static_cast<int>(1LL * B * ((H + 1) / 2) * ((W + 1) / 2));
  const uintptr_t vec = reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(a) |
                        reinterpret_cast<uintptr_t>(da) | reinterpret_cast<uintptr_t>(dl);
  if ((vec & 15) || (reinterpret_cast<uintptr_t>(am) & 7)) return 0;  // vector accesses
  PlbCfg pc;
  if (!(reinterpret_cast<uintptr_t>(am) & 15) && pool_lrn_staged_cfg(B, H, W, C, z, &pc)) {
    int* st = status ? status : aux_status_word();
    if (!st) return 0;
    auto gs = [&](auto kern) {
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pc.smem);
      kern<<<pc.blocks, pc.threads, pc.smem, s>>>(dy, am, a, dl, da, B, H, W, C, z, k, alpha,
                                                  beta, pc.nst, bias_part, st);
    };
    if (z == 3 && H == 55 && W == 55)
      b34 ? gs(k_pool_lrn_bwd_s<3, 55, true>) : gs(k_pool_lrn_bwd_s<3, 55, false>);
    else if (z == 3 && H == 27 && W == 27)
      b34 ? gs(k_pool_lrn_bwd_s<3, 27, true>) : gs(k_pool_lrn_bwd_s<3, 27, false>);
    else
      b34 ? gs(k_pool_lrn_bwd_s<0, 0, true>) : gs(k_pool_lrn_bwd_s<0, 0, false>);
    count_launch();
    return pc.blocks;
  }
  // persistent blocks (at most kPoolLrnBlocks, one bias partial row each)
  if (pool_lrn_use_warp_kernel(C)) {
    auto gw = [&](auto kern) {
      kern<<<blocks, 256, 0, s>>>(dy, am, a, dl, da, nquads, H, W, C, z, k, alpha, beta,
                                  bias_part);
    };
    if (z == 3 && H == 55 && W == 55)
      b34 ? gw(k_pool_lrn_bwd_w<3, 55, true>) : gw(k_pool_lrn_bwd_w<3, 55, false>);
    else if (z == 3 && H == 27 && W == 27)
      b34 ? gw(k_pool_lrn_bwd_w<3, 27, true>) : gw(k_pool_lrn_bwd_w<3, 27, false>);
    else
      b34 ? gw(k_pool_lrn_bwd_w<0, 0, true>) : gw(k_pool_lrn_bwd_w<0, 0, false>);
    count_launch();
    return blocks;
  }
  auto go = [&](auto kern) {
    kern<<<blocks, 256, 0, s>>>(dy, am, a, dl, da, nquads, nq, H, W, C, z, k, alpha, beta,
                                bias_part);
  };
  if (z == 3 && H == 55 && W == 55)
    b34 ? go(k_pool_lrn_bwd<3, 55, true>) : go(k_pool_lrn_bwd<3, 55, false>);
  else if (z == 3 && H == 27 && W == 27)
    b34 ? go(k_pool_lrn_bwd<3, 27, true>) : go(k_pool_lrn_bwd<3, 27, false>);
  else
    b34 ? go(k_pool_lrn_bwd<0, 0, true>) : go(k_pool_lrn_bwd<0, 0, false>);
  count_launch();
  return blocks;
}
int launch_pool_relu_bwd_staged(const bf16* dy, const uint8_t* am, const bf16* a, bf16* da,
                                int B, int H, int W, int C, int z, float* bias_part, int* status,
                                cudaStream_t s) {
  if (C % kSlab || C > 2048 || (z != 2 && z != 3) || H < z || W < z) return 0;
  if (1LL * B * H * W * C >= (1LL << 31)) return 0;  // 32-bit element offsets
  const uintptr_t vec = reinterpret_cast<uintptr_t>(dy) | reinterpret_cast<uintptr_t>(a) |
                        reinterpret_cast<uintptr_t>(da) | reinterpret_cast<uintptr_t>(am);
  PlbCfg pc;
  if ((vec & 15) || !pool_lrn_staged_cfg(B, H, W, C, z, &pc)) return 0;
  int* st = status ? status : aux_status_word();
  if (!st) return 0;
  auto gs = [&](auto kern) {
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, pc.smem);
    kern<<<pc.blocks, pc.threads, pc.smem, s>>>(dy, am, a, nullptr, da, B, H, W, C, z, 0.f, 0.f,
                                                0.f, pc.nst, bias_part, st);
  };
  gs(k_pool_lrn_bwd_s<0, 0, false, false>);
  count_launch();
  return pc.blocks;
}
void launch_pool_fwd_f32(const float* x, float* y, int B, int H, int W, int C, int z, int st,
                         cudaStream_t s) {
  const int Ho = (H - z) / st + 1, Wo = (W - z) / st + 1;
  k_pool_fwd_f32<<<grid_for(1LL * B * Ho * Wo * C, 256), 256, 0, s>>>(x, y, B, H, W, C, z, st);
  count_launch();
}
void launch_fc_finalize(const float* part, int S, int rows, int cols, const float* bias,
                        int relu, int dropout_mode, int layer, const HParams* hp, bf16* out_bf16,
                        float* out_f32, cudaStream_t s) {
  k_fc_finalize<<<grid_for(1LL * rows * cols / 4, 256), 256, 0, s>>>(
      part, S, rows, cols, bias, relu, dropout_mode, layer, hp, out_bf16, out_f32);
  count_launch();
}
void launch_dgrad_finalize(const float* part, int S, int rows, int cols, const bf16* mask,
                           bf16* out, cudaStream_t s) {
  k_dgrad_finalize<<<grid_for(1LL * rows * cols / 8, 256), 256, 0, s>>>(part, S, rows, cols,
                                                                       mask, out);
  count_launch();
}
void launch_dropout_mask(const HParams* hp, int layer, int rows, int cols, uint8_t* keep,
                         cudaStream_t s) {
  k_dropout_mask<<<grid_for(1LL * rows * cols / 4, 256), 256, 0, s>>>(hp, layer, rows, cols,
                                                                     keep);
  count_launch();
}
void launch_softmax_ce(const float* logits, const int32_t* labels, int B, int N, float* probs,
                       bf16* dlogits, float* loss_rows, int* status, cudaStream_t s) {
  k_softmax_ce<<<B, 256, 0, s>>>(logits, labels, B, N, probs, dlogits, loss_rows, status);
  count_launch();
}
void launch_loss_mean(const float* loss_rows, int B, float* out1, float* out2, cudaStream_t s) {
  k_loss_mean<<<1, 256, 0, s>>>(loss_rows, B, out1, out2);
  count_launch();
}
int colsum_chunks(long long rows) {
  const long long per = colsum_rows(rows);
  return static_cast<int>((rows + per - 1) / per);
}
void launch_colsum_partial(const bf16* m, long long rows, int cols, float* partial,
                           cudaStream_t s) {
  const int G = cols / 8;
  const int Gb = G <= 64 ? G : 16;
  k_colsum_partial<<<dim3(colsum_chunks(rows), (G + Gb - 1) / Gb), 256, 0, s>>>(m, rows, cols,
                                                                             partial);
  count_launch();
}
void launch_sgd_conv(float* w, float* v, const float* part, int S, const ConvMap& m, bf16* fwd,
                     bf16* dg, float* grads_out, const HParams* hp, cudaStream_t s) {
  const long long n = 1LL * m.Cout * m.K * m.K * m.Cg;
  if (!m.s2d && !dg && m.Cg % 4 == 0 &&
      ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(v) |
        reinterpret_cast<uintptr_t>(part) | reinterpret_cast<uintptr_t>(grads_out)) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(fwd) & 7) == 0) {
    k_sgd_conv4<<<grid_for(n / 4, 256), 256, 0, s>>>(w, v, part, S, m, fwd, grads_out, hp);
  } else {
    k_sgd_conv<<<grid_for(n, 256), 256, 0, s>>>(w, v, part, S, m, fwd, dg, grads_out, hp);
  }
  count_launch();
}
void launch_sgd_dense(float* w, float* v, const float* g, long long n, bf16* shadow,
                      float* grads_out, const HParams* hp, cudaStream_t s) {
  k_sgd_dense<<<grid_for(n / 4, 256), 256, 0, s>>>(w, v, g, n, shadow, grads_out, hp);
  count_launch();
}
void launch_sgd_bias(float* b, float* v, const float* partial, int chunks, int n, float* grads_out,
                     const HParams* hp, cudaStream_t s) {
  if (n <= 0) return;
  k_sgd_bias<float><<<(n + 31) / 32, dim3(32, 32), 0, s>>>(b, v, partial, chunks, n, grads_out,
                                                          hp);
  count_launch();
}
void launch_sgd_bias_jobs(BiasJobs jobs, const HParams* hp, cudaStream_t s) {
  int blocks = 0;
  for (int k = 0; k < jobs.count; ++k) {
    jobs.j[k].block0 = blocks;
    blocks += (jobs.j[k].n + 31) / 32;
  }
  if (blocks <= 0) return;
  k_sgd_bias_jobs<<<blocks, dim3(32, 32), 0, s>>>(jobs, hp);
  count_launch();
}
void launch_sgd_bias_rows(float* b, float* v, const bf16* g, int rows, int n, float* grads_out,
                          const HParams* hp, cudaStream_t s) {
  if (n <= 0) return;
  k_sgd_bias<bf16><<<(n + 31) / 32, dim3(32, 32), 0, s>>>(b, v, g, rows, n, grads_out, hp);
  count_launch();
}
void launch_conv_shadows(const float* w, const ConvMap& m, bf16* fwd, bf16* dg, cudaStream_t s) {
  const long long n = 1LL * m.Cout * m.K * m.K * m.Cg;
  k_conv_shadows<<<grid_for(n, 256), 256, 0, s>>>(w, m, fwd, dg);
  count_launch();
}
void launch_sgd_range(float* w, float* v, const float* gsum, long long n, float scale, float lr,
                      float momentum, float wd, cudaStream_t s) {
  k_sgd_range<<<grid_for(n, 256), 256, 0, s>>>(w, v, gsum, n, scale, lr, momentum, wd);
  count_launch();
}
void launch_f32_to_bf16(const float* w, bf16* out, long long n, cudaStream_t s) {
  k_f32_to_bf16<<<grid_for(n, 256), 256, 0, s>>>(w, out, n);
  count_launch();
}
void launch_f32_from_bf16(const bf16* in, float* out, long long n, cudaStream_t s) {
  k_f32_from_bf16<<<grid_for(n, 256), 256, 0, s>>>(in, out, n);
  count_launch();
}
void launch_init_normal(float* w, long long n, float stdv, uint64_t seed, uint32_t tag,
                        cudaStream_t s) {
  k_init_normal<<<grid_for((n + 3) / 4, 256), 256, 0, s>>>(
      w, n, stdv, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32), tag);
  count_launch();
}
void launch_fill(float* w, long long n, float value, cudaStream_t s) {
  k_fill<<<grid_for(n, 256), 256, 0, s>>>(w, n, value);
  count_launch();
}
void launch_augment(const uint8_t* src, int B, const float* mean, const float* pca_vec,
                    const float* pca_val, const HParams* hp, bf16* out, cudaStream_t s) {
  k_augment<<<grid_for(1LL * B * ((227 + kAugRows - 1) / kAugRows) * 256, 256), 256, 0, s>>>(
      src, B, mean, pca_vec, pca_val, hp, out);
  count_launch();
}
void launch_tencrop_inputs(const uint8_t* src, int B, const float* mean, bf16* out,
                           cudaStream_t s) {
  k_tencrop_inputs<<<grid_for(1LL * B * 10 * 227 * 256, 256), 256, 0, s>>>(src, B, mean, out);
  count_launch();
}
void launch_tencrop_reduce(const float* probs10, int B, int N, float* probs_avg, int32_t* top5,
                           cudaStream_t s) {
  k_avg_top5<<<B, 256, N * sizeof(float), s>>>(probs10, 10, N, 10LL * N, N, probs_avg, top5);
  count_launch();
}
void launch_ensemble_reduce(const float* probs, int n, int B, int N, float* probs_avg,
                            int32_t* top5, cudaStream_t s) {
  k_avg_top5<<<B, 256, N * sizeof(float), s>>>(probs, n, 1LL * B * N, N, N, probs_avg, top5);
  count_launch();
}
void launch_conv_wt_f32(const float* w, float* wt, int Cout, int K, int Cg, int groups,
                        cudaStream_t s) {
  k_conv_wt_f32<<<grid_for(1LL * Cout * K * K * Cg, 256), 256, 0, s>>>(w, wt, Cout, K, Cg,
                                                                       groups);
  count_launch();
}
void launch_conv_fwd_f32(const float* x, const float* wt, const float* bias, float* y, int B,
                         int H, int W, int Cin, int Cout, int K, int stride, int pad, int groups,
                         int Ho, int Wo, cudaStream_t s) {
  const int Og = Cout / groups, Cg = Cin / groups;
  const long long tiles = 1LL * B * Ho * ((Wo + kTileP - 1) / kTileP);
  size_t smem = static_cast<size_t>(K) * ((kTileP - 1) * stride + K) * Cg * sizeof(float);
  // the warp sums reuse the patch space
  const size_t red = static_cast<size_t>(kConvWarps) * kTileP * 32 * sizeof(float);
  if (smem < red) smem = red;
  if (smem <= 48 * 1024 && tiles < (1LL << 31)) {
    const dim3 grid(static_cast<unsigned>(tiles), (Og + 31) / 32, groups);
    if (Cg % (4 * kConvWarps) == 0)
      k_conv_fwd_f32_tiled<true><<<grid, 32 * kConvWarps, smem, s>>>(
          x, wt, bias, y, H, W, Cin, Cout, K, stride, pad, groups, Ho, Wo);
    else
      k_conv_fwd_f32_tiled<false><<<grid, 32 * kConvWarps, smem, s>>>(
          x, wt, bias, y, H, W, Cin, Cout, K, stride, pad, groups, Ho, Wo);
  } else {
    long long pix = 1LL * B * Ho * Wo;
    dim3 grid(static_cast<unsigned>(pix < 65535 * 4 ? pix : 65535 * 4), (Og + 127) / 128, groups);
    k_conv_fwd_f32<<<grid, 128, 0, s>>>(x, wt, bias, y, B, H, W, Cin, Cout, K, stride, pad,
                                        groups, Ho, Wo);
  }
  count_launch();
}
void launch_fc_fwd_f32(const float* x, const float* w, const float* bias, float* y, int B, int In,
                       int Out, int relu, float scale, cudaStream_t s) {
  const bool v4 = In % 4 == 0 && ((reinterpret_cast<uintptr_t>(x) |
                                    reinterpret_cast<uintptr_t>(w)) & 15) == 0;
  if (v4)
    k_fc_fwd_f32_v4<<<grid_for(1LL * B * Out * 32, 256), 256, 0, s>>>(x, w, bias, y, B, In, Out,
                                                                      relu, scale);
  else
    k_fc_fwd_f32<<<grid_for(1LL * B * Out * 32, 256), 256, 0, s>>>(x, w, bias, y, B, In, Out,
                                                                   relu, scale);
  count_launch();
}

}  // namespace alx

namespace alx {
namespace {
__global__ void k_philox_raw(const uint32_t* __restrict__ ctr, const uint32_t* __restrict__ key,
                             int n, uint32_t* __restrict__ out) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const U4 r = philox4x32_10(U4{ctr[4 * i], ctr[4 * i + 1], ctr[4 * i + 2], ctr[4 * i + 3]},
                               key[2 * i], key[2 * i + 1]);
    out[4 * i] = r.x;
    out[4 * i + 1] = r.y;
    out[4 * i + 2] = r.z;
    out[4 * i + 3] = r.w;
  }
}
}  // namespace
void launch_philox_raw(const uint32_t* ctr, const uint32_t* key, int n, uint32_t* out,
                       cudaStream_t s) {
  k_philox_raw<<<grid_for(n, 256), 256, 0, s>>>(ctr, key, n, out);
  count_launch();
}
}  // namespace alx
