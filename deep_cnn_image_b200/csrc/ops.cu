// ops.cu -- single-operation entry points (alexnet_ops.h).  Each runs the
// same kernel the training step launches for that stage, on caller tensors,
// with caller-provided device scratch.
#include <cstring>

#include "alexnet.h"
#include "alexnet_ops.h"
#include "conv_desc.h"
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
  bf16* fwd = sc.take<bf16>(m.s2d ? static_cast<size_t>(m.Cout) * 576
                               : static_cast<size_t>(m.Cout) * m.K * m.K * m.P);
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
  if (!x || !w || !y || B < 1 || groups < 1 || Cin % groups || Cout % groups)
    return ALEXNET_ERR_INVALID_ARG;
  ConvShape cs{B, H, W, Cin, Cin / groups, Cout / groups, groups, K, pad};
  if (cs.Cg % 8 || cs.Og % 8 || cs.Ho() < 1 || cs.Wo() < 1 || K < 1 || pad < 0)
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  const size_t n = static_cast<size_t>(Cout) * K * K * cs.Cg;
  float* wf = sc.take<float>(n);
  bf16* wg = sc.take<bf16>(static_cast<size_t>(Cout) * cs.Kdim());
  if (!status || !wf || !wg) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  // canonical [Cout][K][K][Cg] -> the GEMM operand [Cout][K*K*P] (zero pads)
  cudaMemsetAsync(wg, 0, 2 * static_cast<size_t>(Cout) * cs.Kdim(), s);
  launch_f32_from_bf16(static_cast<const bf16*>(w), wf, n, s);
  launch_conv_shadows(wf, ConvMap{Cout, K, cs.Cg, groups, 0, cs.P()}, wg, nullptr, s);
  ConvPlan d;
  if (!conv_plan_fwd(&d, cs, x, wg, bias, relu, nullptr, y, num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  return done(conv_plan_launch(d, s));
}

alexnet_status alexnet_op_conv1_fwd(const void* x, int B, const void* w, const float* bias,
                                    void* y, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !w || !y || B < 1 || (reinterpret_cast<uintptr_t>(x) & 15))
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  bf16* xs = sc.take<bf16>(static_cast<size_t>(B) * 57 * 57 * 64);
  float* wf = sc.take<float>(96 * 363);
  bf16* ws2 = sc.take<bf16>(96 * 576);
  if (!status || !xs || !wf || !ws2) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  cudaMemsetAsync(ws2, 0, 2 * 96 * 576, s);
  launch_s2d(static_cast<const bf16*>(x), xs, B, s);
  launch_f32_from_bf16(static_cast<const bf16*>(w), wf, 96 * 363, s);
  launch_conv_shadows(wf, ConvMap{96, 11, 3, 1, 1, 64}, ws2, nullptr, s);
  ConvPlan d;
  if (!conv_plan_fwd(&d, ConvShape{B, 57, 57, 64, 48, 96, 1, 3, 0}, xs, ws2, bias, 1, nullptr, y,
                     num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  return done(conv_plan_launch(d, s));
}

alexnet_status alexnet_op_conv_dgrad(const void* dy, int B, int H, int W, int Cin, const void* w,
                                     int Cout, int K, int pad, int groups, const void* mask,
                                     void* dx, void* ws, size_t ws_bytes, void* stream) {
  // the forward conv maps [H,W,Cin] -> [Ho,Wo,Cout]; its data gradient is a
  // forward conv of dy with the flipped kernel and padding K-1-pad
  if (!dy || !w || !dx || B < 1 || groups < 1 || Cin % groups || Cout % groups)
    return ALEXNET_ERR_INVALID_ARG;
  const int Cg = Cin / groups, Og = Cout / groups;
  const int Ho = H + 2 * pad - K + 1, Wo = W + 2 * pad - K + 1;
  if (Cg % 8 || Og % 8 || Ho < 1 || Wo < 1 || K < 1 || pad < 0) return ALEXNET_ERR_INVALID_ARG;
  // the flipped operand keeps Og channels per tap unpadded
  if (Og % 64 || Ho + 2 * (K - 1 - pad) - K + 1 != H) return ALEXNET_ERR_UNSUPPORTED;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  const size_t n = static_cast<size_t>(Cout) * K * K * Cg;
  const ConvMap m{Cout, K, Cg, groups, 0, 64 * ((Cg + 63) / 64)};
  float* wf = sc.take<float>(n);
  bf16* fwd = sc.take<bf16>(static_cast<size_t>(Cout) * K * K * m.P);
  bf16* dg = sc.take<bf16>(n);
  if (!status || !wf || !fwd || !dg) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_f32_from_bf16(static_cast<const bf16*>(w), wf, n, s);
  launch_conv_shadows(wf, m, fwd, dg, s);
  ConvPlan d;
  if (!conv_plan_dgrad(&d, ConvShape{B, Ho, Wo, Cout, Og, Cg, groups, K, K - 1 - pad}, dy, fwd,
                       m.P, dg, mask, dx, num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  return done(conv_plan_launch(d, s));
}

alexnet_status alexnet_op_conv_wgrad(const void* x, int B, int H, int W, int Cin, const void* dy,
                                     int Cout, int K, int pad, int groups, int splits, float* dw,
                                     void* ws, size_t ws_bytes, void* stream) {
  if (!x || !dy || !dw || B < 1 || groups < 1 || Cin % groups || Cout % groups)
    return ALEXNET_ERR_INVALID_ARG;
  ConvShape cs{B, H, W, Cin, Cin / groups, Cout / groups, groups, K, pad};
  if (cs.Cg % 8 || cs.Og % 8 || cs.Ho() < 1 || cs.Wo() < 1 || K < 1 || pad < 0)
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  ConvPlan d;
  if (!conv_plan_wgrad(&d, cs, x, dy, nullptr, splits, num_sms(), status, true))
    return ALEXNET_ERR_UNSUPPORTED;
  float* part = sc.take<float>(d.f32_need());
  if (!status || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  if (!conv_plan_wgrad(&d, cs, x, dy, part, splits, num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  if (cudaError_t e = conv_plan_launch(d, s)) return done(e);
  return reduce_wgrad(ConvMap{Cout, K, cs.Cg, groups, 0, cs.P()}, part, d.splits(), dw, sc, s);
}

alexnet_status alexnet_op_conv1_wgrad(const void* x, int B, const void* dy, int splits, float* dw,
                                      void* ws, size_t ws_bytes, void* stream) {
  if (!x || !dy || !dw || B < 1 || (reinterpret_cast<uintptr_t>(x) & 15))
    return ALEXNET_ERR_INVALID_ARG;
  Scratch sc(ws, ws_bytes);
  int* status = sc.take<int>(1);
  bf16* xs = sc.take<bf16>(static_cast<size_t>(B) * 57 * 57 * 64);
  const ConvShape cs{B, 57, 57, 64, 48, 96, 1, 3, 0};
  ConvPlan d;
  if (!conv_plan_wgrad(&d, cs, xs, dy, nullptr, splits, num_sms(), status, true))
    return ALEXNET_ERR_UNSUPPORTED;
  float* part = sc.take<float>(d.f32_need());
  if (!status || !xs || !part) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaMemsetAsync(status, 0, 4, s);
  launch_s2d(static_cast<const bf16*>(x), xs, B, s);
  if (!conv_plan_wgrad(&d, cs, xs, dy, part, splits, num_sms(), status))
    return ALEXNET_ERR_UNSUPPORTED;
  if (cudaError_t e = conv_plan_launch(d, s)) return done(e);
  return reduce_wgrad(ConvMap{96, 11, 3, 1, 1, 64}, part, d.splits(), dw, sc, s);
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

alexnet_status alexnet_op_lrn_pool_fwd(const void* a, int B, int H, int W, int C, int z, float k,
                                       float alpha, float beta, void* lo, void* y,
                                       uint8_t* argmax, void* stream) {
  if (!a || !y || !argmax || B < 1 || C < 32 || C % 32 || (z != 2 && z != 3) || H < z || W < z)
    return ALEXNET_ERR_INVALID_ARG;
  if (!launch_lrn_pool_fwd(static_cast<const bf16*>(a), static_cast<bf16*>(lo),
                           static_cast<bf16*>(y), argmax, B, H, W, C, z, k, alpha, beta,
                           static_cast<cudaStream_t>(stream)))
    return ALEXNET_ERR_UNSUPPORTED;
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_pool_lrn_bwd(const void* dy, const uint8_t* argmax, const void* a, int B,
                                       int H, int W, int C, int z, float k, float alpha,
                                       float beta, void* dl, void* da, void* stream) {
  if (!dy || !argmax || !a || !da || B < 1 || C < 32 || C % 32 || (z != 2 && z != 3) || H < z ||
      W < z)
    return ALEXNET_ERR_INVALID_ARG;
  if (!launch_pool_lrn_bwd(static_cast<const bf16*>(dy), argmax, static_cast<const bf16*>(a),
                           static_cast<bf16*>(dl), static_cast<bf16*>(da), B, H, W, C, z, k, alpha,
                           beta, nullptr, nullptr, static_cast<cudaStream_t>(stream)))
    return ALEXNET_ERR_UNSUPPORTED;
  return done(cudaGetLastError());
}

alexnet_status alexnet_op_wait_probe(int* status, long long limit_cycles, void* stream) {
  if (!status || limit_cycles < 1 || limit_cycles > 4000000000LL) return ALEXNET_ERR_INVALID_ARG;
  launch_wait_probe(status, limit_cycles, static_cast<cudaStream_t>(stream));
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
