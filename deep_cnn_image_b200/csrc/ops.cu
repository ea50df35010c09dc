// ops.cu -- single-operation entry points (alexnet_ops.h).  Each runs the
// same kernel the training step launches for that stage, on caller tensors,
// with caller-provided device scratch.
#include <cstring>

#include "alexnet.h"
#include "alexnet_ops.h"
#include "gemm.h"
#include "kernels.h"

using namespace alx;

namespace {

int g_num_sms = 0;

int num_sms() {
  if (!g_num_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

struct Scratch {
  char* base;
  size_t cap, off = 0;
  Scratch(void* b, size_t c) : base(static_cast<char*>(b)), cap(c) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~static_cast<size_t>(255);
    if (!base || off + n * sizeof(T) > cap) return nullptr;
    T* p = reinterpret_cast<T*>(base + off);
    off += n * sizeof(T);
    return p;
  }
};

alexnet_status done(cudaError_t e) { return e == cudaSuccess ? ALEXNET_OK : ALEXNET_ERR_CUDA; }

int pick_bn(int n) {
  if (n == 48 || n == 64 || n == 96 || n == 128 || n == 192 || n == 256) return n;
  if (n % 192 == 0) return 192;
  if (n % 256 == 0) return 256;
  if (n % 128 == 0) return 128;
  return 0;
}
int pick_bn_mn(int n) {
  if (n <= 64) return 64;
  if (n <= 128) return 128;
  if (n % 192 == 0) return 192;
  if (n <= 256 || n % 256 == 0) return 256;
  return 128;
}

struct ConvGeom {
  int H, W, Cin, Cout, K, pad, groups, Ho, Wo;
  int Cg() const { return Cin / groups; }
  int Og() const { return Cout / groups; }
};

bool geom_ok(const ConvGeom& g) {
  return g.H > 0 && g.W > 0 && g.Cin > 0 && g.Cout > 0 && g.K > 0 && g.pad >= 0 && g.groups > 0 &&
         g.Cin % g.groups == 0 && g.Cout % g.groups == 0 && g.Cg() % 8 == 0 && g.Og() % 8 == 0 &&
         g.Ho > 0 && g.Wo > 0;
}

GatherDesc gather_of(const ConvGeom& g, const void* x, int B) {
  GatherDesc d;
  d.src = static_cast<const bf16*>(x);
  d.H = g.H;
  d.W = g.W;
  d.C = g.Cin;
  d.cg_off = g.Cg();
  d.Cg8 = g.Cg() / 8;
  d.KW = g.K;
  d.pad = g.pad;
  d.Ho = g.Ho;
  d.Wo = g.Wo;
  d.Kc = g.K * g.K * g.Cg() / 8;
  d.Mpix = B * g.Ho * g.Wo;
  return d;
}

alexnet_status run_conv_fwd(const ConvGeom& g, const void* x, int B, const bf16* wgemm,
                            const float* bias, int relu, void* y, int* status, cudaStream_t s) {
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_GATHER_K;
  d.bsrc = B_TMA_K;
  d.bn = pick_bn(g.Og());
  if (!d.bn) return ALEXNET_ERR_UNSUPPORTED;
  GemmArgs& a = d.args;
  a.g = gather_of(g, x, B);
  a.M = a.g.Mpix;
  a.N = g.Og();
  a.Kblocks = (a.g.Kc + 7) / 8;
  a.groups = g.groups;
  a.b_goff = g.Og();
  a.epi = EPI_BF16;
  a.relu = relu;
  a.out = y;
  a.ld_out = g.Cout;
  a.col_goff = g.Og();
  a.bias = bias;
  a.status = status;
  const int Kd = g.K * g.K * g.Cg();
  if (!make_tmap_bf16(&d.tmB, wgemm, Kd, g.Cout, 2ull * Kd, 64, d.bn)) return ALEXNET_ERR_INVALID_ARG;
  d.tmA = d.tmB;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  return done(gemm_launch(d, s));
}

alexnet_status run_conv_wgrad(const ConvGeom& g, const void* x, int B, const void* dy, int splits,
                              float* part, int* S_out, int* status, cudaStream_t s) {
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_GATHER_MN;
  d.bsrc = B_TMA_MN;
  d.bn = pick_bn_mn(g.Og());
  GemmArgs& a = d.args;
  a.g = gather_of(g, x, B);
  a.M = g.K * g.K * g.Cg();
  a.N = g.Og();
  a.Kblocks = (a.g.Mpix + 63) / 64;
  a.groups = g.groups;
  a.b_goff = g.Og();
  if (splits <= 0) {
    const long long tiles = 1LL * ((a.M + 127) / 128) * ((a.N + d.bn - 1) / d.bn) * a.groups;
    long long sp = (2LL * num_sms() + tiles - 1) / tiles;
    if (sp > a.Kblocks / 8) sp = a.Kblocks / 8;
    splits = sp < 1 ? 1 : static_cast<int>(sp);
  }
  if (splits > a.Kblocks) splits = a.Kblocks;
  a.kb_per_split = (a.Kblocks + splits - 1) / splits;
  a.epi = EPI_F32_T;
  a.out = part;
  a.ld_out = a.M;
  a.group_stride = 1LL * g.Og() * a.M;
  a.split_stride = 1LL * g.groups * g.Og() * a.M;
  a.status = status;
  if (!make_tmap_bf16(&d.tmB, dy, g.Cout, a.g.Mpix, 2ull * g.Cout, 64, 64))
    return ALEXNET_ERR_INVALID_ARG;
  d.tmA = d.tmB;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  *S_out = d.args.splits;
  return done(gemm_launch(d, s));
}

HParams zero_hp() {
  HParams hp;
  memset(&hp, 0, sizeof(hp));
  return hp;
}

// Sum split-K weight-gradient partials into a canonical-layout gradient with
// the training step's own reduction kernel (an SGD step with lr = 0 whose
// gradient output is kept).
alexnet_status reduce_wgrad(const ConvMap& m, const float* part, int S, float* dw, Scratch& sc,
                            cudaStream_t s) {
  const size_t n = static_cast<size_t>(m.Cout) * m.K * m.K * m.Cg;
  float* w = sc.take<float>(n);
  float* v = sc.take<float>(n);
  bf16* fwd = sc.take<bf16>(m.s2d ? static_cast<size_t>(m.Cout) * 432 : n);
  bf16* dg = m.s2d ? nullptr : sc.take<bf16>(n);
  HParams* hp = sc.take<HParams>(1);
  if (!w || !v || !fwd || (!m.s2d && !dg) || !hp) return ALEXNET_ERR_INVALID_ARG;
  cudaMemsetAsync(w, 0, n * 4, s);
  cudaMemsetAsync(v, 0, n * 4, s);
  launch_write_hparams(hp, zero_hp(), s);
  launch_sgd_conv(w, v, part, S, m, fwd, dg, dw, hp, s);
  return done(cudaGetLastError());
}

}  // namespace

extern "C" {

alexnet_status alexnet_op_conv_fwd(const void* x, int B, int H, int W, int Cin, const void* w,
                                   const float* bias, int Cout, int K, int pad, int groups,
                                   int relu, void* y, void* ws, size_t ws_bytes, void* stream) {
  ConvGeom g{H, W, Cin, Cout, K, pad, groups, H + 2 * pad - K + 1, W + 2 * pad - K + 1};
  if (!x || !w || !y || B < 1 || !geom_ok(g)) return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  if (!status) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  return run_conv_fwd(g, x, B, static_cast<const bf16*>(w), bias, relu, y, status, s);
}

alexnet_status alexnet_op_conv1_fwd(const void* x, int B, const void* w, const float* bias,
                                    void* y, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || B < 1) return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  bf16* xs = sc.take<bf16>(static_cast<size_t>(B) * 57 * 57 * 48);
  float* wf = sc.take<float>(96 * 363);
  bf16* ws2 = sc.take<bf16>(96 * 432);
  if (!status || !xs || !wf || !ws2) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  cudaMemsetAsync(ws2, 0, 2 * 96 * 432, s);
  launch_s2d(static_cast<const bf16*>(x), xs, B, s);
  launch_f32_from_bf16(static_cast<const bf16*>(w), wf, 96 * 363, s);
  ConvMap m{96, 11, 3, 1, 1};
  launch_conv_shadows(wf, m, ws2, nullptr, s);
  ConvGeom g{57, 57, 48, 96, 3, 0, 1, 55, 55};
  return run_conv_fwd(g, xs, B, ws2, bias, 1, y, status, s);
}

alexnet_status alexnet_op_conv_dgrad(const void* dy, int B, int H, int W, int Cin, const void* w,
                                     int Cout, int K, int pad, int groups, const void* mask,
                                     void* dx, void* ws, size_t ws_bytes, void* stream) {
  // the forward conv maps [H,W,Cin] -> [Ho,Wo,Cout]; its data gradient is a
  // forward conv of dy with the flipped kernel and padding K-1-pad
  ConvGeom fw{H, W, Cin, Cout, K, pad, groups, H + 2 * pad - K + 1, W + 2 * pad - K + 1};
  if (!dy || !w || !dx || B < 1 || !geom_ok(fw)) return ALEXNET_ERR_INVALID_ARG;
  ConvGeom g{fw.Ho, fw.Wo, Cout, Cin, K, K - 1 - pad, groups, H, W};
  if (g.Ho != fw.Ho + 2 * g.pad - K + 1 || g.Wo != fw.Wo + 2 * g.pad - K + 1)
    return ALEXNET_ERR_UNSUPPORTED;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  const size_t n = static_cast<size_t>(Cout) * K * K * (Cin / groups);
  float* wf = sc.take<float>(n);
  bf16* fwd = sc.take<bf16>(n);
  bf16* dg = sc.take<bf16>(n);
  if (!status || !wf || !fwd || !dg) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_f32_from_bf16(static_cast<const bf16*>(w), wf, n, s);
  ConvMap m{Cout, K, Cin / groups, groups, 0};
  launch_conv_shadows(wf, m, fwd, dg, s);
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_GATHER_K;
  d.bsrc = B_TMA_K;
  d.bn = pick_bn(g.Og());
  if (!d.bn) return ALEXNET_ERR_UNSUPPORTED;
  GemmArgs& a = d.args;
  a.g = gather_of(g, dy, B);
  a.M = a.g.Mpix;
  a.N = g.Og();
  a.Kblocks = (a.g.Kc + 7) / 8;
  a.groups = groups;
  a.b_goff = g.Og();
  a.epi = mask ? EPI_BF16_MASK : EPI_BF16;
  a.out = dx;
  a.ld_out = Cin;
  a.col_goff = g.Og();
  a.mask = static_cast<const bf16*>(mask);
  a.ld_mask = Cin;
  a.status = status;
  const int Kd = K * K * g.Cg();
  if (!make_tmap_bf16(&d.tmB, dg, Kd, Cin, 2ull * Kd, 64, d.bn)) return ALEXNET_ERR_INVALID_ARG;
  d.tmA = d.tmB;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  return done(gemm_launch(d, s));
}

alexnet_status alexnet_op_conv_wgrad(const void* x, int B, int H, int W, int Cin, const void* dy,
                                     int Cout, int K, int pad, int groups, int splits, float* dw,
                                     void* ws, size_t ws_bytes, void* stream) {
  ConvGeom g{H, W, Cin, Cout, K, pad, groups, H + 2 * pad - K + 1, W + 2 * pad - K + 1};
  if (!x || !dy || !dw || B < 1 || !geom_ok(g)) return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  const int Kb = (B * g.Ho * g.Wo + 63) / 64;
  const int smax = splits > 0 ? (splits < Kb ? splits : Kb) : Kb;
  float* part = sc.take<float>(static_cast<size_t>(smax) * Cout * K * K * g.Cg());
  if (!status || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  int S = 0;
  alexnet_status st = run_conv_wgrad(g, x, B, dy, splits, part, &S, status, s);
  if (st != ALEXNET_OK) return st;
  ConvMap m{Cout, K, g.Cg(), groups, 0};
  return reduce_wgrad(m, part, S, dw, sc, s);
}

alexnet_status alexnet_op_conv1_wgrad(const void* x, int B, const void* dy, int splits, float* dw,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (!x || !dy || !dw || B < 1) return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  bf16* xs = sc.take<bf16>(static_cast<size_t>(B) * 57 * 57 * 48);
  const int Kb = (B * 55 * 55 + 63) / 64;
  const int smax = splits > 0 ? (splits < Kb ? splits : Kb) : Kb;
  float* part = sc.take<float>(static_cast<size_t>(smax) * 96 * 432);
  if (!status || !xs || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_s2d(static_cast<const bf16*>(x), xs, B, s);
  ConvGeom g{57, 57, 48, 96, 3, 0, 1, 55, 55};
  int S = 0;
  alexnet_status st = run_conv_wgrad(g, xs, B, dy, splits, part, &S, status, s);
  if (st != ALEXNET_OK) return st;
  ConvMap m{96, 11, 3, 1, 1};
  return reduce_wgrad(m, part, S, dw, sc, s);
}

alexnet_status alexnet_op_fc_fwd(const void* x, int B, int In, const void* w, int Out, int splits,
                                 float* y, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || B < 1 || In % 8 || Out % 8 || In <= 0 || Out <= 0)
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  HParams* hp = sc.take<HParams>(1);
  const int Kb = (In + 63) / 64;
  if (splits <= 0) splits = Kb >= 16 ? 4 : 1;
  if (splits > Kb) splits = Kb;
  float* part = sc.take<float>(static_cast<size_t>(splits) * B * Out);
  if (!status || !hp || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_write_hparams(hp, zero_hp(), s);
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_TMA_K;
  d.bsrc = B_TMA_K;
  d.bn = 128;
  GemmArgs& a = d.args;
  a.M = B;
  a.N = Out;
  a.Kblocks = Kb;
  a.kb_per_split = (Kb + splits - 1) / splits;
  a.groups = 1;
  a.epi = EPI_F32;
  a.out = part;
  a.ld_out = Out;
  a.split_stride = 1LL * B * Out;
  a.status = status;
  if (!make_tmap_bf16(&d.tmA, x, In, B, 2ull * In, 64, 128) ||
      !make_tmap_bf16(&d.tmB, w, In, Out, 2ull * In, 64, 128))
    return ALEXNET_ERR_INVALID_ARG;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  cudaError_t e = gemm_launch(d, s);
  if (e != cudaSuccess) return ALEXNET_ERR_CUDA;
  launch_fc_finalize(part, d.args.splits, B, Out, nullptr, 0, 0, 6, hp, nullptr, y, s);
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_fc_dgrad(const void* dz, int B, int Out, const void* w, int In,
                                   int splits, float* dx, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (!dz || !w || !dx || B < 1 || In % 64 || Out % 8 || In <= 0 || Out <= 0)
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  HParams* hp = sc.take<HParams>(1);
  const int Kb = (Out + 63) / 64;
  if (splits <= 0) splits = Kb >= 16 ? 4 : 1;
  if (splits > Kb) splits = Kb;
  float* part = sc.take<float>(static_cast<size_t>(splits) * B * In);
  if (!status || !hp || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_write_hparams(hp, zero_hp(), s);
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_TMA_K;
  d.bsrc = B_TMA_MN;
  d.bn = In % 256 == 0 ? 256 : (In % 128 == 0 ? 128 : 64);
  GemmArgs& a = d.args;
  a.M = B;
  a.N = In;
  a.Kblocks = Kb;
  a.kb_per_split = (Kb + splits - 1) / splits;
  a.groups = 1;
  a.epi = EPI_F32;
  a.out = part;
  a.ld_out = In;
  a.split_stride = 1LL * B * In;
  a.status = status;
  if (!make_tmap_bf16(&d.tmA, dz, Out, B, 2ull * Out, 64, 128) ||
      !make_tmap_bf16(&d.tmB, w, In, Out, 2ull * In, 64, 64))
    return ALEXNET_ERR_INVALID_ARG;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  cudaError_t e = gemm_launch(d, s);
  if (e != cudaSuccess) return ALEXNET_ERR_CUDA;
  launch_fc_finalize(part, d.args.splits, B, In, nullptr, 0, 0, 6, hp, nullptr, dx, s);
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_fc_wgrad(const void* dz, const void* x, int B, int Out, int In,
                                   float* dw, void* ws, size_t ws_bytes, void* stream) {
  if (!dz || !x || !dw || B < 1 || In % 64 || Out % 8 || In <= 0 || Out <= 0)
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  if (!status) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  GemmDesc d;
  memset(&d, 0, sizeof(d));
  d.asrc = A_TMA_MN;
  d.bsrc = B_TMA_MN;
  d.bn = In % 256 == 0 ? 256 : (In % 128 == 0 ? 128 : 64);
  GemmArgs& a = d.args;
  a.M = Out;
  a.N = In;
  a.Kblocks = (B + 63) / 64;
  a.kb_per_split = a.Kblocks;
  a.groups = 1;
  a.epi = EPI_F32;
  a.out = dw;
  a.ld_out = In;
  a.status = status;
  if (!make_tmap_bf16(&d.tmA, dz, Out, B, 2ull * Out, 64, 64) ||
      !make_tmap_bf16(&d.tmB, x, In, B, 2ull * In, 64, 64))
    return ALEXNET_ERR_INVALID_ARG;
  if (!gemm_finalize(&d, num_sms())) return ALEXNET_ERR_UNSUPPORTED;
  return done(gemm_launch(d, s));
}

alexnet_status alexnet_op_lrn_fwd(const void* a, int64_t P, int C, float k, float alpha,
                                  float beta, void* b, void* stream) {
  if (!a || !b || P < 1 || C < 8 || C % 8) return ALEXNET_ERR_INVALID_ARG;
  launch_lrn_fwd(static_cast<const bf16*>(a), static_cast<bf16*>(b), P, C, 5, k, alpha, beta,
                 static_cast<cudaStream_t>(stream));
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_lrn_bwd(const void* a, const void* g, int64_t P, int C, float k,
                                  float alpha, float beta, void* da, void* stream) {
  if (!a || !g || !da || P < 1 || C < 8 || C % 8) return ALEXNET_ERR_INVALID_ARG;
  launch_lrn_bwd(static_cast<const bf16*>(a), static_cast<const bf16*>(g), static_cast<bf16*>(da),
                 P, C, 5, k, alpha, beta, static_cast<cudaStream_t>(stream));
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_pool_fwd(const void* x, int B, int H, int W, int C, int z, int st,
                                   void* y, uint8_t* argmax, void* stream) {
  if (!x || !y || !argmax || B < 1 || C % 8 || z < 1 || z > 15 || st < 1 || H < z || W < z)
    return ALEXNET_ERR_INVALID_ARG;
  launch_pool_fwd(static_cast<const bf16*>(x), static_cast<bf16*>(y), argmax, B, H, W, C, z, st,
                  static_cast<cudaStream_t>(stream));
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_pool_bwd(const void* dy, const uint8_t* argmax, const void* pooled,
                                   int B, int H, int W, int C, int z, int st, int relu_mask,
                                   void* dx, void* stream) {
  if (!dy || !argmax || !dx || (relu_mask && !pooled) || B < 1 || C % 8 || z < 1 || z > 15 ||
      st < 1 || H < z || W < z)
    return ALEXNET_ERR_INVALID_ARG;
  launch_pool_bwd(static_cast<const bf16*>(dy), argmax, static_cast<const bf16*>(pooled),
                  static_cast<bf16*>(dx), B, H, W, C, z, st, relu_mask,
                  static_cast<cudaStream_t>(stream));
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_softmax_ce(const float* logits, const int32_t* labels, int B, int N,
                                     float* probs, void* dlogits, float* loss, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (!logits || B < 1 || N < 1) return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  float* rows = sc.take<float>(B);
  if (!status || !rows) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_softmax_ce(logits, labels, B, N, probs, labels ? static_cast<bf16*>(dlogits) : nullptr,
                    rows, status, s);
  if (labels && loss) launch_loss_mean(rows, B, nullptr, loss, s);
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_dropout_mask(uint64_t seed, uint32_t layer, uint32_t step, float p,
                                       int rows, int cols, uint8_t* keep, void* ws,
                                       size_t ws_bytes, void* stream) {
  if (!keep || rows < 1 || cols < 4 || cols % 4 || !(p >= 0.f && p < 1.f))
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  HParams* hp = sc.take<HParams>(1);
  if (!hp) return ALEXNET_ERR_INVALID_ARG;
  HParams v = zero_hp();
  v.step = step;
  v.seed_lo = static_cast<uint32_t>(seed);
  v.seed_hi = static_cast<uint32_t>(seed >> 32);
  v.dropout_p = p;
  const double t = static_cast<double>(p) * 4294967296.0 + 0.5;
  v.drop_thresh = t >= 4294967295.0 ? 0xFFFFFFFFu : static_cast<uint32_t>(t);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  launch_write_hparams(hp, v, s);
  launch_dropout_mask(hp, static_cast<int>(layer), rows, cols, keep, s);
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_philox(const uint32_t* ctr, const uint32_t* key, int n, uint32_t* out,
                                 void* stream) {
  if (!ctr || !key || !out || n < 1) return ALEXNET_ERR_INVALID_ARG;
  launch_philox_raw(ctr, key, n, out, static_cast<cudaStream_t>(stream));
  return done(cudaGetLastError());
}

}  // extern "C"
