// conv_desc.cu -- see conv_desc.h.  The convolution as an implicit GEMM over
// its (kh, kw, cin) taps ("ImageNet Classification with Deep Convolutional
// Neural Networks", summary page, 3.4 "Overall Architecture"; "AlexNet and
// Deep CNNs", "Time complexity of one forward pass").
#include <cstring>

#include "conv_desc.h"

namespace alx {

int conv_pick_bn(int n) {
  if (n == 48 || n == 64 || n == 96 || n == 128 || n == 192 || n == 256) return n;
  if (n % 192 == 0) return 192;
  if (n % 256 == 0) return 256;
  if (n % 128 == 0) return 128;
  return 0;
}

int conv_pick_bn_mn(int n) {
  if (n <= 64) return 64;
  if (n <= 128) return 128;
  if (n % 192 == 0) return 192;
  if (n <= 256 || n % 256 == 0) return 256;
  return 128;
}

static void im2col_geom(GatherDesc* g, const ConvShape& cs) {
  memset(g, 0, sizeof(*g));
  g->H = cs.H;
  g->W = cs.W;
  g->C = cs.C;
  g->cg_off = cs.Cg;
  g->KW = cs.K;
  g->pad = cs.pad;
  g->Ho = cs.Ho();
  g->Wo = cs.Wo();
  g->Mpix = cs.B * cs.Ho() * cs.Wo();
  g->cpt = cs.P() / 64;
  g->Kc = cs.K * cs.K * g->cpt;  // (tap, 64-channel chunk) blocks
}

bool conv_desc_fwd(GemmDesc* d, const ConvShape& cs, const void* x, const void* w,
                   const float* bias, int relu, const void* mask, void* y, int num_sms,
                   int* status, bool dry) {
  memset(d, 0, sizeof(*d));
  if (cs.Cg % 8 || cs.Og % 8 || cs.C % 8 || cs.Ho() < 1 || cs.Wo() < 1) return false;
  d->asrc = A_IM2COL_K;
  d->bsrc = B_TMA_K;
  d->bn = conv_pick_bn(cs.Og);
  if (!d->bn) return false;
  GemmArgs& a = d->args;
  im2col_geom(&a.g, cs);
  a.M = a.g.Mpix;
  a.N = cs.Og;
  a.Kblocks = cs.K * cs.K * a.g.cpt;
  a.groups = cs.groups;
  a.b_goff = cs.Og;
  a.epi = mask ? EPI_BF16_MASK : EPI_BF16;
  a.relu = relu;
  a.out = y;
  a.ld_out = static_cast<long long>(cs.groups) * cs.Og;
  a.col_goff = cs.Og;
  a.bias = bias;
  a.mask = static_cast<const __nv_bfloat16*>(mask);
  a.ld_mask = a.ld_out;
  a.status = status;
  if (!dry) {
    if (!make_tmap_im2col(&d->tmA, x, cs.B, cs.H, cs.W, cs.C, cs.K, cs.pad, 128)) return false;
    const int Kd = cs.Kdim();
    if (!make_tmap_bf16(&d->tmB, w, Kd, static_cast<uint64_t>(cs.groups) * cs.Og,
                        static_cast<uint64_t>(Kd) * 2, 64, d->bn))
      return false;
  }
  return gemm_finalize(d, num_sms);
}

bool conv_desc_wgrad(GemmDesc* d, const ConvShape& cs, const void* x, const void* dy,
                     float* part, int splits, int num_sms, int* status, bool dry) {
  memset(d, 0, sizeof(*d));
  if (cs.Cg % 8 || cs.Og % 8 || cs.C % 8 || cs.Ho() < 1 || cs.Wo() < 1) return false;
  d->asrc = A_IM2COL_MN;
  d->bsrc = B_TMA_MN;
  d->bn = conv_pick_bn_mn(cs.Og);
  GemmArgs& a = d->args;
  im2col_geom(&a.g, cs);
  a.M = cs.Kdim();
  a.N = cs.Og;
  a.Kblocks = (a.g.Mpix + 63) / 64;
  a.groups = cs.groups;
  a.b_goff = cs.Og;
  if (splits <= 0) {
    const long long tiles = 1LL * ((a.M + 127) / 128) * ((a.N + d->bn - 1) / d->bn) * a.groups;
    long long s = (2LL * num_sms + tiles - 1) / tiles;
    if (s > a.Kblocks / 8) s = a.Kblocks / 8;
    splits = s < 1 ? 1 : static_cast<int>(s);
  }
  if (splits > a.Kblocks) splits = a.Kblocks;
  a.kb_per_split = (a.Kblocks + splits - 1) / splits;
  a.epi = EPI_F32_T;
  a.out = part;
  a.ld_out = a.M;
  a.group_stride = 1LL * cs.Og * a.M;
  a.split_stride = 1LL * cs.groups * cs.Og * a.M;
  a.status = status;
  if (!dry) {
    if (!make_tmap_im2col(&d->tmA, x, cs.B, cs.H, cs.W, cs.C, cs.K, cs.pad, 64)) return false;
    const int Cout = cs.groups * cs.Og;
    if (!make_tmap_bf16(&d->tmB, dy, Cout, a.g.Mpix, static_cast<uint64_t>(Cout) * 2, 64, 64))
      return false;
  }
  return gemm_finalize(d, num_sms);
}

size_t ConvPlan::f32_need() const {
  if (box) return b.kind == 1 ? static_cast<size_t>(b.args.splits) * b.args.split_stride : 0;
  const GemmArgs& a = g.args;
  return a.epi == EPI_F32_T ? static_cast<size_t>(a.splits) * a.split_stride : 0;
}

bool conv_plan_fwd(ConvPlan* p, const ConvShape& cs, const void* x, const void* w,
                   const float* bias, int relu, const void* mask, void* y, int num_sms,
                   int* status, bool dry) {
  p->box = box_desc_fwd(&p->b, cs, x, w, bias, relu, mask, y, num_sms, status, dry);
  if (p->box) return true;
  return conv_desc_fwd(&p->g, cs, x, w, bias, relu, mask, y, num_sms, status, dry);
}

bool conv_plan_dgrad(ConvPlan* p, const ConvShape& dg, const void* dy, const void* w_fwd,
                     int p_fwd, const void* w_dg, const void* mask, void* dx, int num_sms,
                     int* status, bool dry) {
  p->box = box_desc_dgrad(&p->b, dg, dy, w_fwd, p_fwd, mask, dx, num_sms, status, dry);
  if (p->box) return true;
  if (!w_dg && !dry) return false;
  return conv_desc_fwd(&p->g, dg, dy, w_dg, nullptr, 0, mask, dx, num_sms, status, dry);
}

bool conv_plan_wgrad(ConvPlan* p, const ConvShape& cs, const void* x, const void* dy,
                     float* part, int splits, int num_sms, int* status, bool dry) {
  p->box = box_desc_wgrad(&p->b, cs, x, dy, part, splits, num_sms, status, dry);
  if (p->box) return true;
  return conv_desc_wgrad(&p->g, cs, x, dy, part, splits, num_sms, status, dry);
}

cudaError_t conv_plan_launch(const ConvPlan& p, cudaStream_t s) {
  return p.box ? box_launch(p.b, s) : gemm_launch(p.g, s);
}

}  // namespace alx
