/*
 * alexnet.h -- C ABI of libalexnet.so: the AlexNet training hot path on one
 * B200 (sm_100a).
 *
 * What the calls compute (pages cited by title and section):
 *   [S] "ImageNet Classification with Deep Convolutional Neural Networks"
 *       (paper-graph-ui summary page);
 *   [W] "AlexNet and Deep CNNs" (fermi.ai wiki page);
 *   [P2] "AlexNet Part 2: Turning the Training Recipe into Testable Design
 *       Choices" (bloss0m page).
 *   - The network: [S] 3.4 "Overall Architecture" and [W] "Layer-by-layer
 *     structure": 227x227x3 input; conv1 96@11x11/s4/p0, conv2 256@5x5/p2,
 *     conv3 384@3x3/p1, conv4 384@3x3/p1, conv5 256@3x3/p1, each + ReLU;
 *     LRN after conv1 and conv2 ([S] 3.4 "Local Response Normalization",
 *     k=2, n=5, alpha=1e-4, beta=0.75); 3x3/s2 max-pool after conv1, conv2
 *     and conv5 ([S] 3.4 "Overlapping Pooling"); FC6 9216->4096, FC7
 *     4096->4096 with ReLU and dropout p=0.5 ([S] 3.4 "Dropout"); FC8
 *     4096->1000 and softmax.  With `grouped`, conv2/conv4/conv5 are
 *     2-group convolutions: the two-GPU restricted connectivity ([S] 3.4
 *     "Training on Multiple GPUs"; [P2] "Reading Figure 2": 5x5x48 and
 *     3x3x192 kernels) run on one GPU.
 *   - The training step: [W] listing TRAIN_STEP and [S] 3.4 "Training
 *     Procedure Details": mean cross-entropy over the batch, backprop,
 *     then for every parameter v <- momentum*v - wd*lr*w - lr*g; w <- w + v.
 *
 * Conventions for every call:
 *   - The caller owns every pointer: inputs, outputs, the workspace and the
 *     stream.  Device pointers must be device memory of the current device;
 *     "host or device" pointers may be either (copies use cudaMemcpyDefault).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default).
 *     Every call is asynchronous on it unless stated; nothing synchronises
 *     the device except alexnet_get_status and host-pointer copies.
 *   - Argument errors are returned before anything is launched.  Errors the
 *     device detects (a label outside [0, 1000), a kernel wait that ran out)
 *     set a sticky status word read by alexnet_get_status.
 *   - No exception crosses the ABI.  alexnet_last_error gives a message.
 *   - Layouts: images NHWC, channels fastest.  Parameters use the canonical
 *     layout of the parameter blob (see alexnet_get_params).
 */
#ifndef ALEXNET_H_
#define ALEXNET_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ALEXNET_API __attribute__((visibility("default")))
#else
#define ALEXNET_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ALEXNET_OK = 0,
  ALEXNET_ERR_INVALID_ARG = 1,  /* bad pointer, size, batch or config value */
  ALEXNET_ERR_UNSUPPORTED = 2,  /* a valid request this build does not serve */
  ALEXNET_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  ALEXNET_ERR_TIMEOUT = 4,      /* a bounded device wait ran out (sticky) */
  ALEXNET_ERR_LABEL_RANGE = 5   /* a label outside [0, 1000) (sticky) */
} alexnet_status;

typedef enum { ALEXNET_FP32 = 0, ALEXNET_BF16 = 1 } alexnet_dtype;
typedef enum { ALEXNET_TRAIN = 0, ALEXNET_INFERENCE = 1 } alexnet_mode;

/* Defaults (alexnet_default_config) are the pages' constants. */
typedef struct {
  int batch_max;          /* largest B any call will use (1 .. 4096) */
  alexnet_dtype dtype;    /* BF16: bf16 operands, fp32 accumulate (train +
                             inference); FP32: fp32 SIMT inference only */
  int grouped;            /* 1: conv2/4/5 have 2 groups (default 1) */
  uint64_t seed;          /* initialisation and Philox key for dropout and
                             augmentation draws */
  float momentum;         /* 0.9 */
  float weight_decay;     /* 5e-4 */
  float dropout_p;        /* 0.5 */
  float lrn_k;            /* 2 */
  float lrn_alpha;        /* 1e-4 (not divided by n) */
  float lrn_beta;         /* 0.75 */
  int lrn_n;              /* 5 (the only size this build serves) */
  int lrn_on;             /* 1; 0 = the no-LRN ablation */
  int pool_size;          /* 3 (overlapping); 2 = non-overlapping ablation */
  int dropout_on;         /* 1; 0 = the no-dropout ablation */
  int keep_grads;         /* 1: keep dL/dparams of the last step for
                             alexnet_get_grads (debug / parity) */
} alexnet_config;

typedef struct alexnet alexnet_t;

/* Fill *cfg with the defaults above (batch_max 128, BF16, grouped). */
ALEXNET_API void alexnet_default_config(alexnet_config* cfg);

/* Number of parameters (weights + biases) of the configured network:
 * 60,965,224 grouped, 62,378,344 ungrouped.  -1 for an invalid config. */
ALEXNET_API int64_t alexnet_param_count(const alexnet_config* cfg);

/* Bytes of device workspace alexnet_create needs for cfg (0 if invalid).
 * Everything the handle uses on the device lives in it: parameters,
 * momentum, bf16 operand copies, activations for batch_max images,
 * gradients and scratch. */
ALEXNET_API size_t alexnet_workspace_bytes(const alexnet_config* cfg);

/* Create a handle over caller-owned device workspace (>= 256-byte aligned,
 * `bytes` >= alexnet_workspace_bytes(cfg)).  Initialises the parameters on
 * `stream` ([S] 3.4 "Training Procedure Details": weights ~ N(0, 0.01^2);
 * biases 1 on conv2, conv4, conv5, FC6, FC7 and 0 on conv1, conv3, FC8),
 * momentum 0 and the step counter 0.  The workspace must stay valid until
 * alexnet_destroy.  *out receives the handle (host memory owned by the
 * library). */
ALEXNET_API alexnet_status alexnet_create(const alexnet_config* cfg, void* workspace, size_t bytes,
                              void* stream, alexnet_t** out);

/* Forward pass of B images (1 <= B <= batch_max).
 *   x:      device, [B,227,227,3] NHWC, bf16 (BF16 handle) or fp32 (FP32),
 *           16-byte aligned.
 *   mode:   ALEXNET_TRAIN draws the dropout masks of the current step
 *           (Philox(seed, step, index)); ALEXNET_INFERENCE keeps every unit
 *           and scales FC6/FC7 outputs by 1 - p ([S] 3.4 "Dropout").
 *   logits: device fp32 [B,1000] (required); probs: device fp32 [B,1000]
 *           softmax, nullable. */
ALEXNET_API alexnet_status alexnet_forward(alexnet_t* h, const void* x, int B, alexnet_mode mode,
                               float* logits, float* probs, void* stream);

/* One training step on B images (BF16 handles only): forward with the
 * step's dropout masks, mean cross-entropy against labels, backward through
 * all eight layers, then the SGD update of every parameter with learning
 * rate lr; the step counter then advances by one.
 *   x:      device bf16 [B,227,227,3], 16-byte aligned;  labels: device int32
 *           [B] in [0,1000)
 *           (an out-of-range label sets ALEXNET_ERR_LABEL_RANGE in the
 *           status word and contributes no loss or gradient);
 *   loss:   device fp32 scalar, nullable: the mean loss of this batch at the
 *           pre-update weights. */
ALEXNET_API alexnet_status alexnet_train_step(alexnet_t* h, const void* x, const int32_t* labels, int B,
                                  float lr, float* loss, void* stream);

/* Training-time augmentation of B source images ([S] 3.4 "Data
 * Augmentation", Forms 1 and 2; mean subtraction [S] 3.2): for image i at
 * the current step, a 224x224 crop at offsets (oy, ox) in 0..31, reflected
 * with probability 1/2, minus the mean image, plus the colour offset
 * [p1 p2 p3][a1 l1, a2 l2, a3 l3]^T with a_j ~ N(0, 0.1^2) drawn once per
 * image; written at the top-left of a 227x227 zero frame.
 *   src: device uint8 [B,256,256,3]; mean: device fp32 [256,256,3];
 *   pca_vec: device fp32 [3][3] row-major, column j = eigenvector p_j;
 *   pca_val: device fp32 [3]; x_out: device bf16 [B,227,227,3]. */
ALEXNET_API alexnet_status alexnet_augment(alexnet_t* h, const uint8_t* src, int B, const float* mean,
                               const float* pca_vec, const float* pca_val, void* x_out,
                               void* stream);

/* Ten-patch test ([S] 3.4 "Data Augmentation", test time): for each of B
 * source images the four corner and the centre 224x224 patches and their
 * reflections (order TL, TR, BL, BR, centre, then reflected), minus the
 * mean image, run through the inference forward; probs_avg is the mean of
 * the ten softmax outputs and top5 the five most probable classes
 * (descending, ties to the lower class index).  BF16 handles only.
 *   src: device uint8 [B,256,256,3]; mean: device fp32 [256,256,3];
 *   probs_avg: device fp32 [B,1000]; top5: device int32 [B,5]. */
ALEXNET_API alexnet_status alexnet_tencrop(alexnet_t* h, const uint8_t* src, int B, const float* mean,
                               float* probs_avg, int32_t* top5, void* stream);

/* Nearest neighbours of feature vectors ([S] "Qualitative Evaluation",
 * Figure 4 right: retrieval by the Euclidean distance between 4096-d
 * last-hidden-layer activations).  For each of Q query rows, the k base rows
 * of smallest squared distance ||q||^2 + ||x||^2 - 2 q.x (the dot products
 * on the tensor cores, fp32 accumulation; negative rounding clamped to 0),
 * ascending, ties to the lower base index.
 *   queries: device bf16 [Q, D]; base: device bf16 [N, D] (both 16-byte
 *   aligned); base_sqnorm: nullable device fp32 [N], the base rows' squared
 *   norms (alexnet_knn_sqnorms); dist: device fp32 [Q, k]; idx: device
 *   int32 [Q, k]; ws: caller-owned device scratch of
 *   alexnet_knn_workspace_bytes(Q, N) bytes (squared norms and per-block
 *   candidate lists, about 10 MB: the Q x N distances are never stored --
 *   the dot-product kernel keeps each query's k best in registers).
 * INVALID_ARG on null pointers, k outside 1..min(32, N), N or D not a
 * multiple of 8, or a scratch too small; UNSUPPORTED if the tensor maps
 * cannot be built (a base pointer not 16-byte aligned). */
ALEXNET_API size_t alexnet_knn_workspace_bytes(int Q, int N);
ALEXNET_API alexnet_status alexnet_knn(const void* queries, int Q, const void* base, int N, int D,
                                       int k, const float* base_sqnorm, float* dist,
                                       int32_t* idx, void* ws, size_t ws_bytes, void* stream);
/* Squared norms of the rows of a device bf16 [rows, D] matrix into a device
 * fp32 [rows] array, the base_sqnorm alexnet_knn accepts (a fixed base needs
 * them once; with base_sqnorm null alexnet_knn computes them every call).
 * INVALID_ARG on null pointers, D not a positive multiple of 8 or x not
 * 16-byte aligned. */
ALEXNET_API alexnet_status alexnet_knn_sqnorms(const void* x, int rows, int D, float* out,
                                               void* stream);

/* Ensemble of networks ([S] "ILSVRC-2012: Single CNN, Ensemble, and
 * Pre-Training Variants": the predictions of several CNNs averaged as the
 * mean of their softmax outputs): each of the n_models handles runs the
 * inference forward on the same batch x, and probs_avg is the mean of their
 * softmax outputs (added in handle order, divided by n_models), top5 its
 * five most probable classes (descending, ties to the lower index).
 *   nets: host array of n_models handles of one dtype, each with
 *   batch_max >= B; x: device [B,227,227,3] in that dtype; probs_avg:
 *   device fp32 [B,1000]; top5: device int32 [B,5]; ws: caller-owned
 *   device scratch of alexnet_ensemble_workspace_bytes(n_models, B) bytes.
 * INVALID_ARG on null pointers, mixed dtypes, B above a handle's batch_max
 * or a scratch too small; otherwise the first failing forward's status. */
ALEXNET_API size_t alexnet_ensemble_workspace_bytes(int n_models, int B);
ALEXNET_API alexnet_status alexnet_ensemble_forward(alexnet_t* const* nets, int n_models,
                                                    const void* x, int B, float* probs_avg,
                                                    int32_t* top5, void* ws, size_t ws_bytes,
                                                    void* stream);

/* Data-parallel training.  The pages train one network split across two
 * GPUs by its channels ([S] 3.4 "Training on Multiple GPUs"); here each
 * GPU holds the whole network and the minibatch is split: each rank computes
 * the gradient of its own images' mean loss, the ranks average the
 * gradients (a reduce-scatter, issued by the caller with its collective
 * library), each rank applies the update of [S] 3.4 "Training Procedure
 * Details" to its own slice of the parameters, and the ranks gather the
 * updated parameters (an all-gather).  The sequence per step:
 *   alexnet_train_grads -> (reduce-scatter of the gradients) ->
 *   alexnet_sgd_range on the rank's slice -> (all-gather of the fp32
 *   parameters into alexnet_device_buffer(h, 0)) -> alexnet_params_updated.
 * The momentum is kept per slice: outside its own slice a rank's momentum
 * values are not updated. */

/* Forward and backward of B images without an update: dL/dparams of the
 * mean loss over these B images into the handle's gradient buffer
 * (alexnet_device_buffer(h, 2); blob order).  image_offset: the index of
 * the first of these images in the whole minibatch; the dropout masks of
 * [S] 3.4 "Dropout" are drawn for those rows of the whole batch, so the
 * ranks together draw exactly the masks one handle would draw for the whole
 * batch.  loss (nullable): device fp32 scalar, the mean over these B images.
 * The FC layers' gradients (the blob from fc6.W on) are complete before the
 * convolutions' backward starts: alexnet_stream_wait_fc_grads lets another
 * stream start reducing them then.  Does not advance the step counter.
 * UNSUPPORTED unless the handle is bf16 and was created with keep_grads. */
ALEXNET_API alexnet_status alexnet_train_grads(alexnet_t* h, const void* x, const int32_t* labels,
                                               int B, int64_t image_offset, float* loss,
                                               void* stream);

/* Makes `stream` wait until the FC gradients of the last alexnet_train_grads
 * are complete (call it after that call; INVALID_ARG before any). */
ALEXNET_API alexnet_status alexnet_stream_wait_fc_grads(alexnet_t* h, void* stream);

/* The update on the parameters [offset, offset + count) of the blob:
 * v <- momentum v - weight_decay lr w - lr (grad_scale gsum); w <- w + v,
 * gsum: device fp32 [count] (the sum of the ranks' gradients of this slice;
 * grad_scale = 1 / ranks gives their mean).  The bf16 operand copies are not
 * refreshed (alexnet_params_updated does that).  INVALID_ARG for a range
 * outside the blob, a null gsum or lr < 0. */
ALEXNET_API alexnet_status alexnet_sgd_range(alexnet_t* h, int64_t offset, int64_t count,
                                             const float* gsum, float grad_scale, float lr,
                                             void* stream);

/* After the fp32 parameters have been replaced in place (all-gathered into
 * alexnet_device_buffer(h, 0)): rebuild the bf16 operand copies the kernels
 * read and advance the step counter. */
ALEXNET_API alexnet_status alexnet_params_updated(alexnet_t* h, void* stream);

/* Device address and element count of one of the handle's fp32 arrays in
 * blob order: which = 0 parameters, 1 momentum, 2 gradients (keep_grads
 * handles).  The arrays live in the caller's workspace.  INVALID_ARG for an
 * unknown or absent array. */
ALEXNET_API alexnet_status alexnet_device_buffer(alexnet_t* h, int which, void** ptr,
                                                 int64_t* count);

/* Size of the parameter blob: n fp32 parameters, n fp32 momentum values,
 * then the uint64 step counter (8n + 8 bytes).  Parameter order: conv1.W
 * conv1.b conv2.W conv2.b ... conv5.b fc6.W fc6.b fc7.W fc7.b fc8.W fc8.b;
 * conv weights [Cout][kh][kw][Cin/groups], FC weights [out][in] with the
 * FC6 input index (h*6 + w)*256 + c. */
ALEXNET_API size_t alexnet_params_bytes(const alexnet_t* h);

/* Copy the blob out to dst (host or device, `bytes` >= the blob size).
 * Stream-ordered; a host dst is complete when the call returns. */
ALEXNET_API alexnet_status alexnet_get_params(alexnet_t* h, void* dst, size_t bytes, void* stream);

/* Replace parameters, momentum and step counter from a blob (host or
 * device) and refresh the bf16 operand copies. */
ALEXNET_API alexnet_status alexnet_set_params(alexnet_t* h, const void* src, size_t bytes, void* stream);

/* dL/dparams of the last train step (keep_grads handles): n fp32 values in
 * blob order, copied to dst (host or device). */
ALEXNET_API alexnet_status alexnet_get_grads(alexnet_t* h, float* dst, size_t n, void* stream);

/* Synchronise the handle's last stream and return the sticky device status
 * (ALEXNET_OK, ALEXNET_ERR_TIMEOUT or ALEXNET_ERR_LABEL_RANGE) or a CUDA
 * error.  Reading it clears nothing. */
ALEXNET_API alexnet_status alexnet_get_status(alexnet_t* h);

/* Message of the last error on this handle (or of the last failed create
 * when h is NULL).  The string is owned by the library. */
ALEXNET_API const char* alexnet_last_error(const alexnet_t* h);

/* Release the handle (NULL is accepted).  The workspace is the caller's. */
ALEXNET_API alexnet_status alexnet_destroy(alexnet_t* h);

#ifdef __cplusplus
}
#endif

#endif /* ALEXNET_H_ */
