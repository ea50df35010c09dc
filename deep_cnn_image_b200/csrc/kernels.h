// kernels.h -- launchers for the memory-bound kernels of the AlexNet step
// (everything that is not a tensor-core GEMM).  All run asynchronously on the
// stream given; sizes are in elements unless stated.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "status.h"

namespace alx {

using bf16 = __nv_bfloat16;

// Device-side hyper-parameters of the current call (read by the kernels so
// that a captured graph stays valid when lr or the step counter change).
struct HParams {
  float lr;
  float momentum;
  float weight_decay;
  float dropout_p;
  uint32_t step;
  uint32_t seed_lo, seed_hi;
  uint32_t drop_thresh;  // keep iff Philox word >= drop_thresh
  uint32_t update;       // 1: apply the update; 0: only write the gradients out
  uint32_t row_offset;   // index of the batch's first image in the whole minibatch (dropout draws)
};

// [S] 3.4 "Training Procedure Details", update rule; [W] listing TRAIN_STEP:
// v <- momentum v - wd lr w - lr g ; w <- w + v, for every parameter.
__device__ __forceinline__ void sgd_one(float& w, float& v, float g, const HParams& hp) {
  const float vn = hp.momentum * v - hp.weight_decay * hp.lr * w - hp.lr * g;
  v = vn;
  w = w + vn;
}

// Canonical conv weight [Cout][K][K][Cg] -> positions in the GEMM layouts.
struct ConvMap {
  int Cout, K, Cg, groups;
  int s2d;  // conv1: forward operand is the space-to-depth [Cout][3][3][64] form
  int P;    // channels per tap in the forward operand and the weight-gradient
            // partials (64 * ceil(Cg / 64); 64 for the space-to-depth form)
};

// Kernels launched by this library so far (all launchers and GEMMs).
int64_t launch_counter();
void count_launch();
void count_launch_n(int64_t n);

// A bounded device wait that nothing completes, limited to limit_cycles
// clocks: it must set the TIMEOUT bit in *status and return (failure
// detection without a fault).
void launch_wait_probe(int* status, long long limit_cycles, cudaStream_t s);
void launch_write_hparams(HParams* hp, HParams v, cudaStream_t s);
void launch_sgd_range(float* w, float* v, const float* gsum, long long n, float scale, float lr,
                      float momentum, float wd, cudaStream_t s);

// x [B,227,227,3] (bf16) -> xs [B,57,57,64]: xs[b,i,j,(dy*4+dx)*3+c] = x[b,4i+dy,4j+dx,c]
// (zero beyond row/column 226, and channels 48..63 zero).
void launch_s2d(const bf16* x, bf16* xs, int B, cudaStream_t s);

// LRN over the channel axis of a [P, C] map (C % 8 == 0).
void launch_lrn_fwd(const bf16* a, bf16* b, long long P, int C, int n, float k, float alpha,
                    float beta, cudaStream_t s);
// da = relu'(a) * dLRN/da^T g
void launch_lrn_bwd(const bf16* a, const bf16* g, bf16* da, long long P, int C, int n, float k,
                    float alpha, float beta, cudaStream_t s);
void launch_lrn_fwd_f32(const float* a, float* b, long long P, int C, int n, float k,
                        float alpha, float beta, cudaStream_t s);

// Max pool z x z / stride st (no padding); argmax = window offset, first max wins.
void launch_pool_fwd(const bf16* x, bf16* y, uint8_t* am, int B, int H, int W, int C, int z,
                     int st, cudaStream_t s);
// dx[b,ih,iw,c] = sum over windows covering it whose argmax names it of dy;
// relu_mask: also zero where the pooled value (= the selected input) is <= 0.
// Returns the number of per-block bias partial rows written to bias_part
// ([rows][C] fp32, column sums of the stored dx), 0 when bias_part is null
// or the shape does not allow them (256 % (C / 8) != 0).
int launch_pool_bwd(const bf16* dy, const uint8_t* am, const bf16* pooled, bf16* dx, int B,
                    int H, int W, int C, int z, int st, int relu_mask, cudaStream_t s,
                    float* bias_part = nullptr);
int pool_bwd_parts(int B, int H, int W, int C);
// Fused normalisation (n = 5) + stride-2 max-pool forward; lo (the
// normalised map) is written only when non-null.  False if C % 32 != 0,
// z not in {2, 3}, or the row tile does not fit in shared memory.
bool launch_lrn_pool_fwd(const bf16* a, bf16* lo, bf16* y, uint8_t* am, int B, int H, int W,
                         int C, int z, float k, float alpha, float beta, cudaStream_t s);
// Fused stride-2 max-pool backward + normalisation backward + ReLU mask
// (a > 0) into da; dl (the normalised map's gradient) written when non-null.
// bias_part (nullable): per-block column sums of the stored da, one row of C
// fp32 per block, at most pool_lrn_bwd_parts(B, H, W, C, z) rows, for the
// conv bias update.  status: the word a bounded wait that runs out sets
// (STATUS_TIMEOUT); null: aux_status_word().  Returns the number of bias
// partial rows (blocks), 0 if the shape or the pointers are not supported.
int launch_pool_lrn_bwd(const bf16* dy, const uint8_t* am, const bf16* a, bf16* dl, bf16* da,
                        int B, int H, int W, int C, int z, float k, float alpha, float beta,
                        float* bias_part, int* status, cudaStream_t s);
// The staged pool backward without a normalisation: da = ReLU'(a) * (dy
// routed to the window choices of the stride-2 pool over a); bias column
// sums as launch_pool_lrn_bwd.  Returns the bias partial rows, 0 if the
// shape or the pointers do not suit it (the caller then uses launch_pool_bwd).
int launch_pool_relu_bwd_staged(const bf16* dy, const uint8_t* am, const bf16* a, bf16* da,
                                int B, int H, int W, int C, int z, float* bias_part, int* status,
                                cudaStream_t s);
// A device status word for single-op calls that have no workspace to hold
// one (never cleared by the library; nullptr if it cannot be looked up).
int* aux_status_word();
int pool_lrn_bwd_parts(int B, int H, int W, int C, int z);
void launch_pool_fwd_f32(const float* x, float* y, int B, int H, int W, int C, int z, int st,
                         cudaStream_t s);

// Sum of split-K partials [S][rows][cols] + bias, then ReLU and dropout
// (train: Philox mask of `layer`; inference: x (1-p)) -> bf16; or fp32 logits.
void launch_fc_finalize(const float* part, int S, int rows, int cols, const float* bias,
                        int relu, int dropout_mode, int layer, const HParams* hp, bf16* out_bf16,
                        float* out_f32, cudaStream_t s);
// Sum of split-K partials -> bf16, zero where mask (bf16, same shape) <= 0.
void launch_dgrad_finalize(const float* part, int S, int rows, int cols, const bf16* mask,
                           bf16* out, cudaStream_t s);
// Dropout keep bits of one layer as bytes (for checks).
void launch_dropout_mask(const HParams* hp, int layer, int rows, int cols, uint8_t* keep,
                         cudaStream_t s);

// Softmax + mean cross-entropy.  probs nullable; dlogits (bf16, nullable) =
// (p - onehot)/B; loss_rows[b] = -log p[label]; labels nullable (inference).
void launch_softmax_ce(const float* logits, const int32_t* labels, int B, int N, float* probs,
                       bf16* dlogits, float* loss_rows, int* status, cudaStream_t s);
void launch_loss_mean(const float* loss_rows, int B, float* out1, float* out2, cudaStream_t s);

// Column sums of a bf16 [rows, cols] matrix in fixed order: partial[chunk][col].
int colsum_chunks(long long rows);
void launch_colsum_partial(const bf16* m, long long rows, int cols, float* partial,
                           cudaStream_t s);

// SGD (v <- m v - wd lr w - lr g; w <- w + v) on one parameter tensor.
// Conv weights: g = sum over S split-K partials [S][groups][Og][Kgemm];
// refreshes the bf16 forward operand (and the flipped data-gradient operand
// when dg != nullptr).  grads_out (nullable) receives g in canonical layout.
void launch_sgd_conv(float* w, float* v, const float* part, int S, const ConvMap& m,
                     bf16* fwd, bf16* dg, float* grads_out, const HParams* hp, cudaStream_t s);
// Dense tensors (FC weights with g[i] contiguous; biases from colsum partials).
void launch_sgd_dense(float* w, float* v, const float* g, long long n, bf16* shadow,
                      float* grads_out, const HParams* hp, cudaStream_t s);
void launch_sgd_bias(float* b, float* v, const float* partial, int chunks, int n,
                     float* grads_out, const HParams* hp, cudaStream_t s);
// Several bias updates from fp32 partial column sums in one launch (the
// conv layers' at the end of the backward pass); block0 is filled in.
struct BiasJob {
  float* b;
  float* v;
  const float* partial;
  int chunks, n;
  float* grads_out;
  int block0;
};
struct BiasJobs {
  BiasJob j[5];
  int count;
};
void launch_sgd_bias_jobs(BiasJobs jobs, const HParams* hp, cudaStream_t s);
// Bias update straight from a short bf16 gradient matrix g [rows][n]: the
// bias gradient is its column sum (the FC layers, rows = batch).
void launch_sgd_bias_rows(float* b, float* v, const bf16* g, int rows, int n, float* grads_out,
                          const HParams* hp, cudaStream_t s);
// Refresh bf16 operands from the fp32 masters (after init / set_params).
void launch_conv_shadows(const float* w, const ConvMap& m, bf16* fwd, bf16* dg, cudaStream_t s);
void launch_f32_to_bf16(const float* w, bf16* out, long long n, cudaStream_t s);

// Weights ~ N(0, std^2) from Philox(seed) + Box-Muller; tag distinguishes tensors.
void launch_init_normal(float* w, long long n, float std, uint64_t seed, uint32_t tag,
                        cudaStream_t s);
void launch_fill(float* w, long long n, float value, cudaStream_t s);

// Augmentation: u8 [B,256,256,3] -> bf16 [B,227,227,3] (crop, flip, -mean, +PCA).
void launch_augment(const uint8_t* src, int B, const float* mean, const float* pca_vec,
                    const float* pca_val, const HParams* hp, bf16* out, cudaStream_t s);
// Ten deterministic crops per source image -> bf16 [B*10,227,227,3] (image-major).
void launch_tencrop_inputs(const uint8_t* src, int B, const float* mean, bf16* out,
                           cudaStream_t s);
// Average of the ten softmaxes per image and top-5 (descending, ties -> lower index).
void launch_tencrop_reduce(const float* probs10, int B, int N, float* probs_avg, int32_t* top5,
                           cudaStream_t s);
// Ensemble: probs holds n models' [B][N] probabilities one after another;
// probs_avg = their mean per image (models added in order), top5 its top 5.
void launch_ensemble_reduce(const float* probs, int n, int B, int N, float* probs_avg,
                            int32_t* top5, cudaStream_t s);

// fp32 SIMT forward path.
void launch_conv_wt_f32(const float* w, float* wt, int Cout, int K, int Cg, int groups,
                        cudaStream_t s);
void launch_conv_fwd_f32(const float* x, const float* wt, const float* bias, float* y, int B,
                         int H, int W, int Cin, int Cout, int K, int stride, int pad, int groups,
                         int Ho, int Wo, cudaStream_t s);
void launch_fc_fwd_f32(const float* x, const float* w, const float* bias, float* y, int B,
                       int In, int Out, int relu, float scale, cudaStream_t s);
void launch_f32_from_bf16(const bf16* in, float* out, long long n, cudaStream_t s);
// Raw Philox blocks: out[4i..] = Philox(ctr[4i..], key[2i..]).
void launch_philox_raw(const uint32_t* ctr, const uint32_t* key, int n, uint32_t* out,
                       cudaStream_t s);

}  // namespace alx
