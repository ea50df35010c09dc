// conv_shape.h -- the geometry of one stride-1 convolution launch.
#pragma once

namespace alx {

struct ConvShape {
  int B, H, W;   // input batch and spatial size (stride 1, output = H + 2 pad - K + 1)
  int C;         // channels per input pixel (all groups)
  int Cg;        // input channels per group
  int Og;        // output channels per group
  int groups;
  int K, pad;
  int Ho() const { return H + 2 * pad - K + 1; }
  int Wo() const { return W + 2 * pad - K + 1; }
  int P() const { return 64 * ((Cg + 63) / 64); }  // padded channels per tap
  int Kdim() const { return K * K * P(); }
};

}  // namespace alx
