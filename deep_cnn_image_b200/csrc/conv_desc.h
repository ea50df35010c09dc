// conv_desc.h -- GEMM descriptors of the stride-1 convolutions (forward,
// data gradient as a forward convolution of dY, weight gradient), fed by TMA
// im2col loads.  Shared by the network planner and the single-op entry points.
//
// GEMM K layout of a convolution with Cg input channels per group: taps
// (kh, kw) in row-major order, each tap padded to P = 64 * ceil(Cg / 64)
// channels (k = tap * P + c).  Channels Cg .. P-1 of a tap read either zeros
// (beyond the tensor) or the next group's channels; their weights are zero.
#pragma once
#include "conv_box.h"
#include "conv_shape.h"
#include "gemm.h"

namespace alx {


// Output channel tile for N output channels per group (0 if none fits).
int conv_pick_bn(int n);
int conv_pick_bn_mn(int n);

// y[b, oh, ow, g*Og + o] = epilogue(sum_k im2col(x)[m, k] * w[g*Og + o][k]); w is
// [groups*Og][K*K*P] bf16.  Epilogue: bias + ReLU (mask == nullptr, relu) or
// zero where mask[b, oh, ow, ...] <= 0 (mask != nullptr, for data gradients).
// dry: size the plan without encoding tensor maps (no device needed).
bool conv_desc_fwd(GemmDesc* d, const ConvShape& cs, const void* x, const void* w,
                   const float* bias, int relu, const void* mask, void* y, int num_sms,
                   int* status, bool dry = false);

// Split-K weight gradient: part[s][g][o][k] = sum over the pixels of slice s
// of dy[p, g*Og + o] * im2col(x)[p, k], k over K*K*P.  splits <= 0: automatic.
bool conv_desc_wgrad(GemmDesc* d, const ConvShape& cs, const void* x, const void* dy,
                     float* part, int splits, int num_sms, int* status, bool dry = false);

// One convolution launch: the shifted-box kernel where the shape fits it,
// else the im2col GEMM.
struct ConvPlan {
  bool box = false;
  GemmDesc g;
  BoxDesc b;
  int splits() const { return box ? b.args.splits : g.args.splits; }
  // fp32 scratch (elements) the launch writes: weight-gradient partials
  size_t f32_need() const;
};

bool conv_plan_fwd(ConvPlan* p, const ConvShape& cs, const void* x, const void* w,
                   const float* bias, int relu, const void* mask, void* y, int num_sms,
                   int* status, bool dry = false);
// Data gradient: the box kernel reading the forward weights transposed
// when the shape allows, else the im2col GEMM on the flipped copy w_dg
// (which may then not be null).
bool conv_plan_dgrad(ConvPlan* p, const ConvShape& dg, const void* dy, const void* w_fwd,
                     int p_fwd, const void* w_dg, const void* mask, void* dx, int num_sms,
                     int* status, bool dry = false);
bool conv_plan_wgrad(ConvPlan* p, const ConvShape& cs, const void* x, const void* dy,
                     float* part, int splits, int num_sms, int* status, bool dry = false);
cudaError_t conv_plan_launch(const ConvPlan& p, cudaStream_t s);

}  // namespace alx
