// gemm.h -- host-side description of one tensor-core GEMM launch.
//
// Every convolution (forward, data gradient, weight gradient) and every
// fully-connected product of the network is one launch of the same
// tcgen05 kernel, described by a GemmDesc.  D[M x N] (+)= A[M x K] * B[N x K]^T
// accumulates in fp32 tensor memory; K is walked in 64-element blocks.
//
// Operand sources:
//   A_TMA_K / A_TMA_MN : A read by TMA from a dense bf16 matrix that is
//                        K-contiguous (rows = M) or M-contiguous (rows = K).
//   A_IM2COL_K         : implicit im2col of an NHWC bf16 map by TMA im2col
//                        loads: row m is an output pixel, its K entries the
//                        (kh, kw, cin) taps of one group (stride-1 conv).
//   A_IM2COL_MN        : the transpose of that matrix (rows are output
//                        pixels = the reduction, columns the conv taps), for
//                        weight gradients.
//   B_TMA_K / B_TMA_MN : B read by TMA, K-contiguous (rows = N) or
//                        N-contiguous (rows = K).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace alx {

struct HParams;

enum ASrc : int {
  A_TMA_K = 0,
  A_TMA_MN = 1,
  A_IM2COL_K = 4,   // conv operand by TMA im2col: rows = output pixels, 64 channels of one tap
  A_IM2COL_MN = 5,  // its transpose for weight gradients: rows = pixels (the reduction)
};
enum BSrc : int { B_TMA_K = 0, B_TMA_MN = 1 };
enum Epi : int {
  EPI_BF16 = 0,       // out_bf16[row, col] = act(acc + bias[col])
  EPI_BF16_MASK = 1,  // out_bf16[row, col] = acc if mask[row, col] > 0 else 0
  EPI_F32 = 2,        // out_f32[split][group][row, col] = acc
  EPI_F32_T = 3,      // out_f32[split][group][col, row] = acc
  EPI_SGD_T = 4,      // acc[row, col] = dL/dw of the parameter at col * ld_out + row: the
                      // update applied in place (one split, one group)
};

struct GatherDesc {           // im2col geometry of a stride-1 convolution
  int H, W, C;               // C = channels per pixel (row length in elements)
  int cg_off;                // channel offset of group g is g * cg_off
  int KW, pad;               // kernel width, zero padding (stride 1)
  int Ho, Wo;                // output map size
  int Kc;                    // number of (tap, 64-channel chunk) blocks
  int Mpix;                  // B * Ho * Wo
  int cpt;                   // 64-channel chunks per tap (K = taps * cpt * 64)
};

struct GemmArgs {
  int M, N;           // output extent (rows, columns) of one group
  int Kblocks;        // 64-wide blocks of the reduction
  int kb_per_split;   // blocks per split-K slice
  int splits, groups;
  int m_tiles, n_tiles;
  int a_goff, b_goff;  // per-group coordinate offsets of the TMA operands (in M / N)
  GatherDesc g;
  // epilogue
  int epi;
  int relu;
  void* out;
  long long ld_out;        // elements between rows (cols for EPI_F32_T)
  long long split_stride;  // elements between split-K slices
  long long group_stride;  // elements between groups (F32 modes)
  int col_goff;            // column offset per group (BF16 modes)
  const float* bias;       // nullable, indexed by col + g * col_goff
  const __nv_bfloat16* mask;
  long long ld_mask;
  // EPI_SGD_T: fp32 parameters and momentum updated in place, their bf16
  // copy refreshed, the raw gradient stored when sgd_grads is non-null
  float* sgd_w;
  float* sgd_v;
  __nv_bfloat16* sgd_shadow;
  float* sgd_grads;
  const HParams* hp;
  int* status;
};

struct GemmDesc {
  int asrc, bsrc, bn;
  CUtensorMap tmA, tmB;
  GemmArgs args;
  int grid;
  int smem;
  int stages;
};

// Build a 2-D bf16 tensor map with 128-byte swizzle: `inner` contiguous
// elements per row, `outer` rows `row_bytes` apart, box of box_inner x
// box_outer elements.  Returns false if the driver rejects it.
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

// 4-D tiled tensor map over an NHWC bf16 tensor [N, H, W, C] (dimensions in
// (C, W, H, N) order), box box_c x box_w x box_h x 1, 128-byte swizzle
// (box_c * 2 <= 128).  Out-of-range box elements read as zero.
bool make_tmap_bf16_4d(CUtensorMap* m, const void* base, int C, int W, int H, int N,
                       uint32_t box_c, uint32_t box_w, uint32_t box_h);

// im2col tensor map over an NHWC bf16 tensor [N, H, W, C] for a stride-1
// K x K convolution with zero padding `pad` (both sides): 64 channels per
// pixel, `pixels` pixels per load, 128-byte swizzle.
bool make_tmap_im2col(CUtensorMap* m, const void* base, int N, int H, int W, int C, int K,
                      int pad, int pixels);

// Fill grid/smem/stages of a descriptor whose asrc/bsrc/bn/args are set.
// Returns false for an unsupported combination.
bool gemm_finalize(GemmDesc* d, int num_sms);

// Set the kernels' shared-memory attribute once (before any stream capture).
cudaError_t gemm_prepare();

cudaError_t gemm_launch(const GemmDesc& d, cudaStream_t stream);

}  // namespace alx
