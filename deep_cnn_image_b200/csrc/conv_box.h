// conv_box.h -- stride-1 convolutions whose activation operand is one TMA
// box per 64-channel chunk, reused by every filter tap.
//
// An output tile is To_h whole output rows of one image.  Its input box is
// the (To_h + K - 1)-row, (Wo + K - 1)-pixel window of the zero-padded input
// (TMA fills the padding), 64 channels, laid out as 128-byte rows: box row
// r * Wb + c holds input pixel (oh0 - pad + r, c - pad).  Output position
// m = r * Wb + c of the tile reads, for tap (kh, kw), box row
// m + kh * Wb + kw: the tap's GEMM operand is the box itself, started
// kh * Wb + kw rows further on.  tcgen05 matrix descriptors take such a
// start address directly (the 128-byte swizzle follows the absolute shared
// memory address), so a chunk is loaded once for all K * K taps instead of
// once per tap as with im2col.  Positions c >= Wo of each row are computed
// and dropped.
//
//   forward / data gradient: D[m, n] = sum_{tap, c} box[m + shift(tap), c] W[n][tap, c]
//     M = positions (NSUB sub-tiles of 128), N = output channels, K-major.
//   weight gradient: D[(tap, c), o] = sum_m box[m + shift(tap), c] dY[m, o]
//     M = two taps x 64 channels (the two 64-row halves of the operand are the
//     same box at the two taps' shifts), N = output channels, K = positions;
//     both operands MN-major.  Partial sums per position split, reduced later.
#pragma once
#include "conv_shape.h"
#include "gemm.h"

namespace alx {

struct BoxArgs {
  int B, Ho, Wo;   // output map (forward) / dY map (weight gradient)
  int K, pad;      // kernel size, zero padding of the input
  int Wb;          // box width: Wo + K - 1
  int To_h;        // output rows per tile
  int Hb;          // input rows per box
  int tiles_img;   // ceil(Ho / To_h)
  int cpt;         // 64-channel chunks per tap
  int k16_last;    // 16-channel K steps of the last chunk that hold real channels (forward)
  int cg_off;      // input channel offset of group g: g * cg_off
  int groups;
  int Og;          // output channels per group
  int n_tiles;     // BN-wide tiles over Og
  int sw_n;        // swapped tiles: MMA N = the tile's positions rounded up to 16 (<= 256)
  // forward epilogue (as GemmArgs)
  int epi, relu;
  void* out;
  long long ld_out;
  int col_goff;
  const float* bias;
  const __nv_bfloat16* mask;
  long long ld_mask;
  // data gradient from the forward weights (B operand MN-major): the
  // forward kernel's output channels per group and padded channels per tap
  int w_og, w_p;
  // weight gradient
  int npairs;           // ceil(K * K / 2) tap pairs
  int tsets;            // items the pairs are split over
  int splits;           // position splits
  int tiles_per_split;  // position tiles per split
  int rows_pad;         // K rows (positions) per position tile, multiple of 64
  int P;                // padded channels per tap in the partial sums
  long long split_stride, group_stride;
  float* part;
  int* status;
};

struct BoxDesc {
  // 0: forward / data gradient, 1: weight gradient, 2: data gradient from the
  // forward weights, 3: forward with swapped operands (M = 128 output channels,
  // N = the tile's positions), 4: kind 2 swapped (M = 64 or 128 input channels),
  // 5: kind 4 with two taps of a kernel row on M = 128 (64 input channels at
  // most; a weight stage is one kernel row of 64-channel slabs)
  int kind;
  int bn;
  int nsub;  // forward: 128-row sub-tiles per tile; weight gradient: pairs per item
  CUtensorMap tmX, tmW;  // weight gradient: tmW maps dY
  BoxArgs args;
  int grid, smem;
  int stages_a, stages_b;  // weight gradient: stages_a only
  int a_bytes, b_bytes;    // per-stage shared memory of each ring (forward: b_bytes per tap)
  int tps;                 // forward: taps per weight stage
};

// Forward (or data gradient as a forward convolution of dY): same meaning as
// conv_desc_fwd.  False if the shape does not fit the kernel.
bool box_desc_fwd(BoxDesc* d, const ConvShape& cs, const void* x, const void* w,
                  const float* bias, int relu, const void* mask, void* y, int num_sms,
                  int* status, bool dry = false);

// Data gradient of a forward convolution, as the forward convolution of dy
// (shape dg: the dgrad geometry, channels of dy in, input channels out) with
// the kernel flipped, reading the forward weight operand w_fwd
// ([groups * dg.Cg][K * K * p_fwd], p_fwd = padded input channels per tap of
// the forward convolution) transposed, so no flipped copy is needed.
// Requires dg.Cg % 64 == 0.  mask as in box_desc_fwd.
bool box_desc_dgrad(BoxDesc* d, const ConvShape& dg, const void* dy, const void* w_fwd,
                    int p_fwd, const void* mask, void* dx, int num_sms, int* status,
                    bool dry = false);

// Weight gradient into split partial sums, same layout as conv_desc_wgrad:
// part[s][g][o][tap * P + c].  splits <= 0: automatic.  Returns the split
// count used in d->args.splits.
bool box_desc_wgrad(BoxDesc* d, const ConvShape& cs, const void* x, const void* dy,
                    float* part, int splits, int num_sms, int* status, bool dry = false);

cudaError_t box_prepare();
cudaError_t box_launch(const BoxDesc& d, cudaStream_t stream);

}  // namespace alx
