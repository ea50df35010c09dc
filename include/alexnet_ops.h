/*
 * alexnet_ops.h -- single-operation entry points of libalexnet.so.
 *
 * Each call runs exactly one stage of the network's hot path (the same
 * kernels alexnet_train_step launches) on caller-provided tensors, so that a
 * test can feed the oracle the very inputs the kernel saw.  All pointers are
 * device pointers owned by the caller; `ws` is caller-owned device scratch
 * of `ws_bytes` (a call returns ALEXNET_ERR_INVALID_ARG if it is too small);
 * `stream` is a cudaStream_t as void*.  Calls are asynchronous.  Layouts are
 * NHWC with channels fastest; channel counts must be multiples of 8.
 * Pages cited as in alexnet.h ([S], [W]).
 */
#ifndef ALEXNET_OPS_H_
#define ALEXNET_OPS_H_

#include <stddef.h>
#include <stdint.h>

#include "alexnet.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Stride-1 convolution with zero padding, bias and ReLU ([S] 3.4 "Overall
 * Architecture"), on the tensor cores:
 *   y[b,oh,ow,o] = relu(bias[o] + sum x[b,oh-pad+kh,ow-pad+kw,g*Cg+ci] w[o,kh,kw,ci])
 * x bf16 [B,H,W,Cin]; w bf16 [Cout][K][K][Cin/groups]; bias fp32 [Cout]
 * (nullable); y bf16 [B,Ho,Wo,Cout].  relu 0/1.  Output channels per group
 * must be one of 48, 64, 96, 128, 192, 256 or split into 192/128/256 tiles. */
ALEXNET_API alexnet_status alexnet_op_conv_fwd(const void* x, int B, int H, int W, int Cin, const void* w,
                                   const float* bias, int Cout, int K, int pad, int groups,
                                   int relu, void* y, void* ws, size_t ws_bytes, void* stream);

/* conv1 of the network: 11x11, stride 4, no padding, on a [B,227,227,3]
 * input (computed as a 3x3 stride-1 convolution of its 4x4 space-to-depth
 * form).  x 16-byte aligned; w bf16 [96][11][11][3]; y bf16 [B,55,55,96] =
 * relu(conv + bias). */
ALEXNET_API alexnet_status alexnet_op_conv1_fwd(const void* x, int B, const void* w, const float* bias,
                                    void* y, void* ws, size_t ws_bytes, void* stream);

/* Data gradient of a stride-1 convolution:
 *   dx[b,ih,iw,c] = sum_{o,kh,kw} dy[b,ih+pad-kh,iw+pad-kw,o] w[o,kh,kw,c-g*Cg]
 * (o in c's group), then zeroed where mask[b,ih,iw,c] <= 0 if mask != NULL
 * (mask = the ReLU output that fed this convolution).  dy bf16 [B,H',W',Cout];
 * dx bf16 [B,H,W,Cin] (H' = H for the layers here). */
ALEXNET_API alexnet_status alexnet_op_conv_dgrad(const void* dy, int B, int H, int W, int Cin,
                                     const void* w, int Cout, int K, int pad, int groups,
                                     const void* mask, void* dx, void* ws, size_t ws_bytes,
                                     void* stream);

/* Weight gradient of a stride-1 convolution (fp32 out, canonical layout):
 *   dw[o,kh,kw,ci] = sum_{b,oh,ow} dy[b,oh,ow,o] x[b,oh-pad+kh,ow-pad+kw,g*Cg+ci]
 * split into `splits` K-slices (0 = automatic) summed in a fixed order. */
ALEXNET_API alexnet_status alexnet_op_conv_wgrad(const void* x, int B, int H, int W, int Cin,
                                     const void* dy, int Cout, int K, int pad, int groups,
                                     int splits, float* dw, void* ws, size_t ws_bytes,
                                     void* stream);

/* The same weight gradient without caller scratch and without allocating:
 * for callers that can neither pass this library scratch memory nor let it
 * allocate device memory (for instance code running after a framework has
 * reserved the whole device through its own allocator, or a service that
 * forbids device allocation once it has started).  Arguments as in
 * alexnet_op_conv_wgrad, minus ws/ws_bytes.  The split-K partial sums live
 * in a 16 MiB array in this library's own device memory, which every GPU
 * that loads the library holds until the process exits.  Its device address
 * is looked up (cudaGetSymbolAddress) on the first call on each device, so
 * that first call should come before any stream capture; the look-up is
 * repeated when the device's context has changed (after cudaDeviceReset).
 * All calls share the array: calls whose work overlaps on the GPU race and
 * must be ordered by the caller.  Returns ALEXNET_ERR_UNSUPPORTED when even
 * one K-slice of partial sums (Cout * K * K * roundup(Cin/groups, 64)
 * floats: the channels of a tap are padded to a multiple of 64) exceeds the
 * array; splits is reduced to what the array holds.  The call waits for its
 * own work before it returns (it reads back the kernel's status word): on
 * ALEXNET_OK dw holds the result; ALEXNET_ERR_TIMEOUT means a bounded wait
 * inside the kernel ran out and dw is not valid.  The pages have no
 * counterpart: this is an integration convenience, not part of the method. */
ALEXNET_API alexnet_status alexnet_op_conv_wgrad_noalloc(const void* x, int B, int H, int W,
                                                         int Cin, const void* dy, int Cout, int K,
                                                         int pad, int groups, int splits,
                                                         float* dw, void* stream);

/* conv1 weight gradient on a [B,227,227,3] input (16-byte aligned): dw fp32
 * [96][11][11][3]. */
ALEXNET_API alexnet_status alexnet_op_conv1_wgrad(const void* x, int B, const void* dy, int splits,
                                      float* dw, void* ws, size_t ws_bytes, void* stream);

/* Fully-connected products (fp32 out, no bias):
 *   fwd:   y[b,o]  = sum_i x[b,i] w[o,i]      x bf16 [B,In], w bf16 [Out,In]
 *   dgrad: dx[b,i] = sum_o dz[b,o] w[o,i]     dz bf16 [B,Out]
 *   wgrad: dw[o,i] = sum_b dz[b,o] x[b,i]
 * In and Out must be multiples of 8. */
ALEXNET_API alexnet_status alexnet_op_fc_fwd(const void* x, int B, int In, const void* w, int Out,
                                 int splits, float* y, void* ws, size_t ws_bytes, void* stream);
ALEXNET_API alexnet_status alexnet_op_fc_dgrad(const void* dz, int B, int Out, const void* w, int In,
                                   int splits, float* dx, void* ws, size_t ws_bytes,
                                   void* stream);
ALEXNET_API alexnet_status alexnet_op_fc_wgrad(const void* dz, const void* x, int B, int Out, int In,
                                   float* dw, void* ws, size_t ws_bytes, void* stream);

/* LRN over channels ([S] 3.4 "Local Response Normalization", n = 5):
 * b = a / (k + alpha * sum_{|j-i|<=2} a_j^2)^beta; bwd gives
 * da = relu'(a) * (dLRN/da)^T g.  a, b, g, da bf16 [P, C]. */
ALEXNET_API alexnet_status alexnet_op_lrn_fwd(const void* a, int64_t P, int C, float k, float alpha,
                                  float beta, void* b, void* stream);
ALEXNET_API alexnet_status alexnet_op_lrn_bwd(const void* a, const void* g, int64_t P, int C, float k,
                                  float alpha, float beta, void* da, void* stream);

/* Max pool z x z, stride st, no padding ([S] 3.4 "Overlapping Pooling"):
 * y bf16 [B,Ho,Wo,C] and argmax uint8 (window offset dy*z+dx of the first
 * maximum in row-major order).  bwd routes dy to the argmax of every window
 * (overlaps add); relu_mask zeroes windows whose pooled value is <= 0. */
ALEXNET_API alexnet_status alexnet_op_pool_fwd(const void* x, int B, int H, int W, int C, int z, int st,
                                   void* y, uint8_t* argmax, void* stream);
ALEXNET_API alexnet_status alexnet_op_pool_bwd(const void* dy, const uint8_t* argmax, const void* pooled,
                                   int B, int H, int W, int C, int z, int st, int relu_mask,
                                   void* dx, void* stream);

/* Normalisation (n = 5) then stride-2 max-pooling, fused ([S] 3.4 "Local
 * Response Normalization" and "Overlapping Pooling"; pooling follows the
 * normalisation after conv1 and conv2): a bf16 [B,H,W,C] (post-ReLU conv
 * output), y bf16 [B,Ho,Wo,C] and argmax uint8 [B,Ho,Wo,C] as
 * alexnet_op_pool_fwd produces them from alexnet_op_lrn_fwd's output
 * (bit-identical); lo (nullable) receives that normalised map [B,H,W,C].
 * Ho = (H - z)/2 + 1.  C % 32 == 0, z in {2, 3}, W small enough that
 * 10 rows x W x 32 bf16 channels fit in 48 KB (W <= 76); else
 * ALEXNET_ERR_INVALID_ARG / ALEXNET_ERR_UNSUPPORTED. */
ALEXNET_API alexnet_status alexnet_op_lrn_pool_fwd(const void* a, int B, int H, int W, int C,
                                                   int z, float k, float alpha, float beta,
                                                   void* lo, void* y, uint8_t* argmax,
                                                   void* stream);

/* Backward of alexnet_op_lrn_pool_fwd and of the ReLU below it, fused: dy
 * bf16 [B,Ho,Wo,C] pooled-map gradient, argmax from the forward, a the
 * forward's input; da bf16 [B,H,W,C] = ReLU'(a) * LRN-backward(a,
 * pool-backward(dy, argmax)); dl (nullable) receives the pool-backward
 * result (the normalised map's gradient).  Same shape rules as the
 * forward, and C <= 2048. */
ALEXNET_API alexnet_status alexnet_op_pool_lrn_bwd(const void* dy, const uint8_t* argmax,
                                                   const void* a, int B, int H, int W, int C,
                                                   int z, float k, float alpha, float beta,
                                                   void* dl, void* da, void* stream);

/* Softmax + cross-entropy over N classes: probs fp32 [B,N] (nullable),
 * dlogits bf16 [B,N] = (p - onehot)/B (nullable), loss fp32 scalar (mean).
 * labels device int32 [B] (nullable: no loss, no dlogits). */
ALEXNET_API alexnet_status alexnet_op_softmax_ce(const float* logits, const int32_t* labels, int B, int N,
                                     float* probs, void* dlogits, float* loss, void* ws,
                                     size_t ws_bytes, void* stream);

/* Dropout keep mask (uint8 0/1, [rows, cols]) of FC `layer` (6 or 7) at
 * `step` with key `seed` and drop probability p ([S] 3.4 "Dropout"): kept
 * iff word (e & 3) of Philox4x32-10((e >> 2, layer, step, 0), seed) >=
 * round(p * 2^32), e = row*cols + col. */
ALEXNET_API alexnet_status alexnet_op_dropout_mask(uint64_t seed, uint32_t layer, uint32_t step, float p,
                                       int rows, int cols, uint8_t* keep, void* ws,
                                       size_t ws_bytes, void* stream);

/* Raw Philox4x32-10 blocks on the device: for i < n, out[4i..4i+3] =
 * Philox(ctr[4i..4i+3], key[2i..2i+1]).  ctr, key, out device uint32. */
ALEXNET_API alexnet_status alexnet_op_philox(const uint32_t* ctr, const uint32_t* key, int n, uint32_t* out,
                                 void* stream);

/* Which kernel runs convolution `layer` (0..4) for a batch of `batch`
 * images: pass 0 forward, 1 data gradient (layers 1..4), 2 weight gradient.
 * *algo = 1: the shifted-box kernel (one input box per 64-channel chunk for
 * all filter taps), 0: the im2col GEMM. */
ALEXNET_API alexnet_status alexnet_conv_algo(alexnet_t* h, int batch, int layer, int pass,
                                             int* algo);

/* keep != 0: later forward and training calls also store the normalised
 * maps after conv1/conv2 and their gradients (debug_copy 10/11, 70/71), at
 * the cost of the extra writes; results are otherwise identical.  Default 0.
 * The pages have no counterpart (a debugging aid). */
ALEXNET_API alexnet_status alexnet_debug_keep(alexnet_t* h, int keep);

/* Failure detection without a fault: one device thread waits on an
 * mbarrier that nothing completes, through the same bounded wait the
 * pipelined kernels use, limited to limit_cycles SM clocks (1 ..
 * 4,000,000,000).  When the limit runs out the wait ORs the TIMEOUT bit (1)
 * into *status (a caller-owned device int) and the kernel returns; the
 * context stays usable.  The pages have no counterpart (a reliability
 * check).  INVALID_ARG for a null status or a limit out of range. */
ALEXNET_API alexnet_status alexnet_op_wait_probe(int* status, long long limit_cycles,
                                                 void* stream);

/* fused != 0 (default): the FC weight-gradient GEMM applies the SGD update
 * ([S] "ImageNet Classification with Deep Convolutional Neural Networks",
 * 3.4 "Training Procedure Details") to the FC weights in its epilogue, so
 * no fp32 weight gradient reaches memory.  0: the gradient goes to scratch
 * and a separate kernel applies the same update.  Results are identical;
 * the switch exists to compare the two. */
ALEXNET_API alexnet_status alexnet_debug_fc_update(alexnet_t* h, int fused);

/* on != 0 (default): in a training step each conv layer's weight gradient and
 * update run on a second stream of the handle beside the data-gradient chain
 * (forked once the layer's output gradient is complete; the update waits
 * for the data gradient that reads the layer's old bf16 weights; joined
 * before the step ends), so the two fill each other's idle SMs.  0: one
 * stream.  Results are bit-identical; the switch exists to compare the two.
 * While stats_enable is on the step runs on one stream either way, so that
 * every GEMM is timed alone. */
ALEXNET_API alexnet_status alexnet_debug_overlap(alexnet_t* h, int on);

/* Bounds evidence without a sanitiser: every buffer the handle carves out of
 * its workspace is followed by a 256-byte guard region, filled with the byte
 * 0xA5 by alexnet_create.  This call synchronises the handle's last stream
 * and stores in *bad_bytes how many guard bytes no longer hold 0xA5: 0
 * unless some kernel wrote past the end of a workspace buffer.  INVALID_ARG
 * for a null handle or pointer.  The pages have no counterpart (a debugging
 * aid). */
ALEXNET_API alexnet_status alexnet_debug_canaries(alexnet_t* h, int64_t* bad_bytes);

/* One internal tensor of the handle's last forward (debug / parity):
 * which = 0..4 conv l+1 output after ReLU, 10/11 LRN1/LRN2 output,
 * 20/21/24 pool1/pool2/pool5 output, 30/31 FC6/FC7 output after dropout,
 * 40 logits (fp32); gradients of the last training step (bf16):
 * 50+l dL/d(pre-activation of conv l+1), 60+l dL/d(pooled map after conv
 * l+1), 70+l dL/d(LRN output of conv l+1), 80 dL/dlogits, 81/82 dL/d(FC7/FC6
 * pre-activation); 90/91/94 the uint8 window choices (argmax) of the pools
 * after conv1/conv2/conv5.  Copies min(bytes, tensor bytes) to dst (host or
 * device).  10/11 and 70/71 hold data only for calls made with
 * alexnet_debug_keep(h, 1): normalisation and pooling run as one fused
 * kernel that otherwise keeps the normalised map and its gradient on chip. */
ALEXNET_API alexnet_status alexnet_debug_copy(alexnet_t* h, int which, void* dst, size_t bytes,
                                  void* stream);

/* Launch accounting and GEMM timing of a handle's calls.  While enabled,
 * every tensor-core GEMM launch of alexnet_train_step / alexnet_forward is
 * bracketed by CUDA events on the call's stream (inside a replayed CUDA graph
 * as event nodes of that graph).  alexnet_stats_read synchronises that stream
 * and fills *out for the most recent such call (zeros if none since enabling):
 *   launches:      kernels this library launched for it
 *   gemm_launches: of which tensor-core GEMMs
 *   gemm_flops:    algorithmic FLOPs of those GEMMs (2 x multiply-adds of
 *                  the network's own layer shapes, padding not counted)
 *   gemm_ms:       summed device time of those GEMM launches */
typedef struct {
  int64_t launches;
  int64_t gemm_launches;
  double gemm_flops;
  double gemm_ms;
} alexnet_stats;

ALEXNET_API alexnet_status alexnet_stats_enable(alexnet_t* h, int enable);
ALEXNET_API alexnet_status alexnet_stats_read(alexnet_t* h, alexnet_stats* out);

/* The i-th GEMM launch (launch order, 0 <= i < gemm_launches) of the call
 * alexnet_stats_read reports: *kind 0 = a convolution (forward, data or
 * weight gradient), 1 = an FC forward or data gradient, 2 = an FC weight
 * gradient written to memory; *flops its algorithmic FLOPs; *ms its device
 * time.  Synchronises that call's stream; ALEXNET_ERR_INVALID_ARG past the
 * last launch. */
ALEXNET_API alexnet_status alexnet_stats_launch(alexnet_t* h, int i, int* kind, double* flops,
                                               double* ms);

#ifdef __cplusplus
}
#endif

#endif /* ALEXNET_OPS_H_ */
