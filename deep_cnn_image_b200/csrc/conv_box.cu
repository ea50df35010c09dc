// conv_box.cu -- the shifted-box convolution kernels (see conv_box.h).
//
// The operation is the stride-1 convolution of "ImageNet Classification
// with Deep Convolutional Neural Networks" (summary page, 3.4 "Overall
// Architecture"; "AlexNet and Deep CNNs", "Time complexity of one forward
// pass"): a sum over the (kh, kw, cin) taps, here ordered chunk by chunk of
// 64 input channels, tap by tap within a chunk.
//
// Both kernels are persistent (one 352-thread CTA per SM): warps 0-7 drain
// tensor memory (epilogue; warps w and w + 4 share TMEM lane quarter w and
// split its 16-column chunks), warp 8 issues TMA loads, warp 9 issues
// tcgen05 MMAs and owns the tensor memory.  Where a tile has two independent
// accumulators (two position sub-tiles, two tap pairs), warp 10 issues the
// second one's MMAs: the per-stage hand-over of each issuing thread (about
// 400 clocks of waits, fences, commits and loop control, measured on B200)
// then runs in parallel instead of adding up in one thread.  Every mbarrier wait is bounded; on
// expiry the kernel records a timeout in the status word and winds down.
#include <cudaTypedefs.h>

#include <cstring>

#include "conv_box.h"
#include "kernels.h"
#include "ptx.cuh"

namespace alx {

namespace {

constexpr int kThreads = 352;
constexpr int kSmemBudget = 227 * 1024;
constexpr int kBarBytes = 3072;  // mbarriers, tmem slot, abort flag (first 512 B); staged bias
constexpr int kMaxBias = (kBarBytes - 512) / 4;
// swapped tiles: per epilogue warp, a staging area for one 32-position chunk
// of 32 bf16 channels, after the barrier block
constexpr int kStageWarp = 32 * 32 * 2;
constexpr int kStageBytes = 8 * kStageWarp;

__host__ __device__ constexpr int pow2_cols(int n) {
  return n <= 32 ? 32 : (n <= 64 ? 64 : (n <= 128 ? 128 : (n <= 256 ? 256 : 512)));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Zero the operand rings once: rows of a stage that no box ever writes are
// read by the MMA (for positions that are dropped) and must hold finite
// values.
__device__ __forceinline__ void zero_smem(uint8_t* p, int bytes) {
  for (int i = threadIdx.x * 16; i < bytes; i += kThreads * 16)
    *reinterpret_cast<uint4*>(p + i) = make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------- forward
// Tile t = ((g * B + b) * tiles_img + ti) * n_tiles + n_t: output rows
// ti * To_h .. of image b, output channels n_t * BN .. of group g.
// SW = 1 swaps the roles: M = the BN (128, or 64 for a data gradient read
// from the forward weights) output channels (the weight slab is the A
// operand), N = the tile's box positions, a.sw_n <= 256 (the shifted box is
// the B operand), so one MMA does BN x sw_n x 16 instead of two
// 128 x BN x 16 ones; the accumulator holds channels in its lanes and
// positions in its columns.  With M = 64, accumulator row r sits in lane
// 32 * (r / 16) + r % 16.  SW = 2 (data gradient, at most 64 input
// channels): M = 128 holds two taps of a kernel row, (kh, 2p) in rows 0-63
// and (kh, 2p + 1) in rows 64-127 (the MN-major weight slabs one after the
// other, the odd last tap beside a zero slab), both multiplied by the box at
// the first tap's shift; the second tap's partial sum for position c then
// sits in column c + 1, and the epilogue adds the two halves.  That halves
// the MMAs an M = 64 tile needs for the same channels.  KT = 10 * K + taps
// per weight stage selects a copy whose tap loop is unrolled for that kernel
// size and stage width (0: both at run time).
template <int BN, int NSUB, int BMN, int SW = 0, int KT = 0>
__global__ void __launch_bounds__(kThreads, 1)
    conv_box_fwd(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                 const __grid_constant__ BoxArgs a, int stA, int stB, int a_bytes, int tps) {
  constexpr int B_BYTES = BN * 128;  // one tap's weight slab; a B stage holds tps of them
  constexpr int ACC_COLS = SW ? 128 * NSUB : NSUB * BN;
  constexpr int ACC_BUFS = (2 * ACC_COLS <= 512) ? 2 : 1;
  constexpr int TMEM_COLS = pow2_cols(ACC_BUFS * ACC_COLS);
  static_assert(!BMN || BN % 64 == 0, "MN-major weights come in 64-channel blocks");
  static_assert(!SW || (NSUB == 2 && (BN == 128 || (BN == 64 && BMN))),
                "swapped tiles: 128 (or 64 MN-major) channels x up to 256 positions");
  static_assert(SW != 2 || (BN == 64 && BMN && KT == 0),
                "tap pairs: 64-channel MN-major slabs, generic tap loop");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + stA * a_bytes;
  // a tap-pair tile's stage is one kernel row, padded to an even number of
  // slabs: the last odd tap pairs with a slab of zeros that no load writes
  const int b_stage = (SW == 2 ? ((a.K + 1) & ~1) : tps) * B_BYTES;
  uint8_t* barp = smem + stA * a_bytes + stB * b_stage;
  const uint32_t a_full = smem_u32(barp);
  const uint32_t a_empty = a_full + 8 * stA;
  const uint32_t b_full = a_empty + 8 * stA;
  const uint32_t b_empty = b_full + 8 * stB;
  const uint32_t acc_full = b_empty + 8 * stB;
  const uint32_t acc_empty = acc_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barp + 8 * (2 * stA + 2 * stB + 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // MMA warps: two where the tile's two sub-tile accumulators are separate
  constexpr int NMW = (NSUB == 2 && !SW) ? 2 : 1;
  zero_smem(smem, stA * a_bytes + (SW == 2 ? stB * b_stage : 0));
  if (threadIdx.x == 0) {
    for (int s = 0; s < stA; ++s) {
      mbar_init(a_full + 8 * s, 1);
      mbar_init(a_empty + 8 * s, NMW);
    }
    for (int s = 0; s < stB; ++s) {
      mbar_init(b_full + 8 * s, 1);
      mbar_init(b_empty + 8 * s, NMW);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + 8 * i, NMW);
      mbar_init(acc_empty + 8 * i, 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total = a.n_tiles * a.tiles_img * a.B * a.groups;
  const int taps = a.K * a.K;
  const uint32_t box_bytes = static_cast<uint32_t>(a.Hb) * a.Wb * 128;
  // the layer's bias, staged once (read by every epilogue chunk)
  float* sbias = reinterpret_cast<float*>(barp + 512);
  if (a.bias && a.epi == EPI_BF16) {
    for (int i = threadIdx.x; i < a.groups * a.col_goff; i += blockDim.x) sbias[i] = a.bias[i];
  }
  __syncthreads();

  if (warp == 8) {
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmW);
      RingPos ra, rb;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        int q = t;
        const int n_t = q % a.n_tiles;
        q /= a.n_tiles;
        const int ti = q % a.tiles_img;
        q /= a.tiles_img;
        const int b = q % a.B;
        const int g = q / a.B;
        const int oh0 = ti * a.To_h;
        for (int ch = 0; ch < a.cpt && ok; ++ch, ra.next(stA)) {
          const int s = ra.slot;
          if (!mbar_wait(a_empty + 8 * s, ra.phase ^ 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(a_full + 8 * s, box_bytes);
          tma_load_4d(sA + s * a_bytes, &tmX, g * a.cg_off + ch * 64, -a.pad, oh0 - a.pad, b,
                      a_full + 8 * s);
          for (int tap0 = 0; tap0 < taps; tap0 += tps, rb.next(stB)) {
            const int sb = rb.slot;
            const int n = min(tps, taps - tap0);
            if (!mbar_wait(b_empty + 8 * sb, rb.phase ^ 1, a.status, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(b_full + 8 * sb, n * B_BYTES);
            for (int j = 0; j < n; ++j) {
              const uint32_t dst = sB + sb * b_stage + j * B_BYTES;
              if (BMN) {
                // forward weight rows g * w_og + ch * 64 .. (64 dy channels),
                // columns of the flipped tap, output channels n_t * BN ..
                const int tapf = taps - 1 - (tap0 + j);
#pragma unroll
                for (int q = 0; q < BN / 64; ++q)
                  tma_load_2d(dst + q * 8192, &tmW, tapf * a.w_p + n_t * BN + 64 * q,
                              g * a.w_og + ch * 64, b_full + 8 * sb);
              } else {
                tma_load_2d(dst, &tmW, ((tap0 + j) * a.cpt + ch) * 64, g * a.Og + n_t * BN,
                            b_full + 8 * sb);
              }
            }
          }
        }
      }
    }
  } else if (warp == 9 || warp == 10) {
    // ---------------------------------------------------------------- MMA
    // Descriptors are built once and advanced by adding 16-byte units to
    // their start-address field: a single issuing thread cannot afford to
    // rebuild two 64-bit descriptors per MMA.  With two MMA warps, warp
    // 9 + mw issues sub-tile mw's MMAs.
    const int mw = warp - 9;
    if (lane == 0 && mw < NMW) {
      const uint32_t IDESC = SW == 2 ? idesc_bf16(128, a.sw_n, 1, 0)
                             : (SW ? idesc_bf16(BN, a.sw_n, BMN, 0) : idesc_bf16(128, BN, 0, BMN));
      const uint64_t adesc0 = smem_desc_sw128(sA, 16, 1024);
      const uint64_t bdesc0 = BMN ? smem_desc_sw128(sB, 8192, 1024) : smem_desc_sw128(sB, 16, 1024);
      const uint32_t a_lo0 = static_cast<uint32_t>(adesc0), a_hi = static_cast<uint32_t>(adesc0 >> 32);
      const uint32_t b_lo0 = static_cast<uint32_t>(bdesc0), b_hi = static_cast<uint32_t>(bdesc0 >> 32);
      const uint32_t a_units = static_cast<uint32_t>(a_bytes) >> 4;
      const uint32_t row_adv = static_cast<uint32_t>(a.Wb - a.K + 1) * 8;  // next kernel row
      // unrolled taps: the box offset of each kernel row, 16-byte units
      constexpr int KR = KT ? KT / 10 : 1;
      uint32_t rowoff[KR];
#pragma unroll
      for (int kh = 0; kh < KR; ++kh) rowoff[kh] = static_cast<uint32_t>(kh * a.Wb) * 8;
      RingPos ra, rb;
      uint32_t tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tcount) {
        const int acc = ACC_BUFS == 2 ? (tcount & 1) : 0;
        const uint32_t aph = ACC_BUFS == 2 ? ((tcount >> 1) & 1) : (tcount & 1);
        if (!mbar_wait(acc_empty + 8 * acc, aph ^ 1, a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t dbase = tmem_base + acc * ACC_COLS;
        for (int ch = 0; ch < a.cpt && ok; ++ch, ra.next(stA)) {
          const int s = ra.slot;
          if (!mbar_wait(a_full + 8 * s, ra.phase, a.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t abox = a_lo0 + s * a_units;
          // a last chunk of 48 real channels (conv1's space-to-depth input,
          // conv2's 48 channels per group) skips the K step of zeros
          const bool k3 = !BMN && ch == a.cpt - 1 && a.k16_last == 3;
          // the MMAs of one tap: A / B at the tap's box shift and weight slab
          auto issue = [&](uint32_t shift, uint32_t bj, uint32_t acc0) {
            if (SW) {
              // A = the tap's weight slab (K-major, or MN-major for the data
              // gradient), B = the box at the tap's shift
              if (k3)
                tc_mma_k3<2, 2>(dbase, bj, b_hi, abox + shift, a_hi, IDESC, acc0);
              else
                tc_mma_k4<BMN ? 128 : 2, 2>(dbase, bj, b_hi, abox + shift, a_hi, IDESC, acc0);
            } else if (NSUB == 2) {
              // this warp's sub-tile: rows 128 mw .. of the box, its own
              // accumulator
              const uint32_t am = abox + shift + mw * (128 * 128 / 16);
              if (k3)
                tc_mma_k3<2, 2>(dbase + mw * BN, am, a_hi, bj, b_hi, IDESC, acc0);
              else
                tc_mma_k4<2, BMN ? 128 : 2>(dbase + mw * BN, am, a_hi, bj, b_hi, IDESC, acc0);
            } else {
              if (k3)
                tc_mma_k3<2, 2>(dbase, abox + shift, a_hi, bj, b_hi, IDESC, acc0);
              else
                tc_mma_k4<2, BMN ? 128 : 2>(dbase, abox + shift, a_hi, bj, b_hi, IDESC, acc0);
            }
          };
          if constexpr (KT == 0) {
            uint32_t shift = 0;  // (kh * Wb + kw) rows, in 16-byte units
            int kw = 0;
            for (int tap0 = 0; tap0 < taps; tap0 += tps, rb.next(stB)) {
              const int sb = rb.slot;
              const int n = min(tps, taps - tap0);
              if (!mbar_wait(b_full + 8 * sb, rb.phase, a.status, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t bst = b_lo0 + sb * (b_stage >> 4);
              if constexpr (SW == 2) {
                // one kernel row per stage (tap0 = kh * K): pair p = taps
                // (kh, 2p) and (kh, 2p + 1) as the two 64-row halves of
                // M (the descriptor's leading offset is one slab), both
                // against the box at the first tap's shift
                const uint32_t srow = static_cast<uint32_t>((tap0 / a.K) * a.Wb) * 8;
                for (int p = 0; 2 * p < a.K; ++p)
                  tc_mma_k4<128, 2>(dbase, bst + 2 * p * (B_BYTES >> 4), b_hi,
                                    abox + srow + 16 * p, a_hi, IDESC,
                                    (ch == 0 && tap0 == 0 && p == 0) ? 0u : 1u);
              } else {
                for (int j = 0; j < n; ++j) {
                  issue(shift, bst + j * (B_BYTES >> 4), (ch == 0 && tap0 + j == 0) ? 0u : 1u);
                  if (++kw == a.K) {
                    kw = 0;
                    shift += row_adv;
                  } else {
                    shift += 8;
                  }
                }
              }
              tc_commit(b_empty + 8 * sb);
            }
          } else {
            // K x K taps in stages of TP, unrolled: every tap's shift and
            // slab offset is a constant plus its kernel row's offset, so the
            // issuing thread spends its time on MMAs rather than on loop
            // bookkeeping (each instruction of that single thread is on the
            // critical path between two stages' MMAs)
            constexpr int KK = KT / 10, TP = KT % 10, NT = KK * KK;
#pragma unroll
            for (int st = 0; st < (NT + TP - 1) / TP; ++st) {
              const int sb = rb.slot;
              if (!mbar_wait(b_full + 8 * sb, rb.phase, a.status, abort_flag)) {
                ok = false;
                break;
              }
              tc_fence_after();
              const uint32_t bst = b_lo0 + sb * (b_stage >> 4);
#pragma unroll
              for (int j = 0; j < TP; ++j) {
                const int tap = st * TP + j;
                if (tap < NT)
                  issue(rowoff[tap / KK] + (tap % KK) * 8, bst + j * (B_BYTES >> 4),
                        (tap == 0 && ch == 0) ? 0u : 1u);
              }
              tc_commit(b_empty + 8 * sb);
              rb.next(stB);
            }
          }
          if (!ok) break;
          tc_commit(a_empty + 8 * s);
        }
        if (!ok) break;
        tc_commit(acc_full + 8 * acc);
      }
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- epilogue
    uint32_t tcount = 0;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tcount) {
      int q = t;
      const int n_t = q % a.n_tiles;
      q /= a.n_tiles;
      const int ti = q % a.tiles_img;
      q /= a.tiles_img;
      const int b = q % a.B;
      const int g = q / a.B;
      const int oh0 = ti * a.To_h;
      const int acc = ACC_BUFS == 2 ? (tcount & 1) : 0;
      const uint32_t aph = ACC_BUFS == 2 ? ((tcount >> 1) & 1) : (tcount & 1);
      // (a tap-pair tile's warps meet at named barriers, so every warp runs
      // every tile even after a timeout; it only stops storing)
      const bool got = mbar_wait(acc_full + 8 * acc, aph, a.status, abort_flag);
      if (!got && SW != 2) break;
      tc_fence_after();
      const int quarter = warp & 3, half = warp >> 2;
      if constexpr (SW == 2) {
        // TMEM lanes 0-63 hold taps (kh, 2p) summed over p: input channel
        // = lane, column = position.  Lanes 64-127 hold taps (kh, 2p + 1),
        // read at the first tap's shift, so their column c belongs to
        // position c - 1: dx[c] = low[c] + high[c + 1].  A high warp
        // (quarter 2, 3) hands columns c0 + 1 .. c0 + 16 to the low warp
        // of the same half (quarter 0, 1) through its staging area; the
        // low warp adds, transposes through its own and stores 16-byte
        // vectors of eight channels.
        const bool high = quarter >= 2;
        const uint32_t pair_bar = 1u + static_cast<uint32_t>(quarter & 1) + 2u * half;
        float* U = reinterpret_cast<float*>(barp + kBarBytes + (warp | 2) * kStageWarp);
        uint8_t* stg = barp + kBarBytes + warp * kStageWarp;
        const int nw = (quarter & 1) * 32;  // the pair's first channel
        const long long cg0 = static_cast<long long>(g) * a.col_goff + nw;
        const uint32_t tb =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
        for (int c0 = 128 * half; c0 < 128 * half + 128 && c0 < a.sw_n; c0 += 16) {
          if (high) {
            float v[32];
            if (c0 + 32 <= ACC_COLS) {
              tmem_ld32(tb + c0, v);
            } else {
              float w16[16];
              tmem_ld16(tb + c0, w16);
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = w16[e];
#pragma unroll
              for (int e = 16; e < 32; ++e) v[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) U[e * 32 + lane] = v[e + 1];
            named_bar_sync(pair_bar, 64);  // handed over
            named_bar_sync(pair_bar, 64);  // taken
          } else {
            float v[16];
            tmem_ld16(tb + c0, v);
            named_bar_sync(pair_bar, 64);
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] += U[e * 32 + lane];
            named_bar_sync(pair_bar, 64);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              reinterpret_cast<__nv_bfloat16*>(stg)[e * 32 + lane] = __float2bfloat16_rn(v[e]);
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 2; ++i) {
              const int j = lane + 32 * i;
              const int e = j >> 2, part = j & 3;
              const int c = c0 + e;
              const int r = c / a.Wb;
              const int col = c - r * a.Wb;
              const int oh = oh0 + r;
              if (got && r < a.To_h && oh < a.Ho && col < a.Wo && nw + part * 8 < a.Og) {
                const uint4 val = *reinterpret_cast<const uint4*>(stg + e * 64 + part * 16);
                *reinterpret_cast<uint4*>(
                    out + ((static_cast<long long>(b) * a.Ho + oh) * a.Wo + col) * a.ld_out +
                    cg0 + part * 8) = val;
              }
            }
            __syncwarp();
          }
        }
      } else if constexpr (SW) {
        // lane = output channel, columns = positions: this warp's CW = 32
        // (M = 64: 16) channels at the 128 positions of its half, 32
        // positions per chunk.  A chunk goes through the warp's staging
        // area transposed (position-major rows of CW bf16 channels), so the
        // global stores are 16-byte vectors of eight channels.
        constexpr int CW = BN == 64 ? 16 : 32;
        constexpr int PIECES = CW / 8;  // 16-byte pieces per position
        const int nw = n_t * BN + quarter * CW;  // the warp's first channel
        const int n = nw + lane;
        const bool cvalid = lane < CW && n < a.Og;
        const float bv = (a.bias && cvalid) ? sbias[static_cast<long long>(g) * a.col_goff + n] : 0.f;
        uint8_t* stg = barp + kBarBytes + warp * kStageWarp;
        const long long cg0 = static_cast<long long>(g) * a.col_goff + nw;
        const uint32_t tb =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS;
#pragma unroll 1
        for (int c0 = 128 * half; c0 < 128 * half + 128 && c0 < a.sw_n; c0 += 32) {
          float v[32];
          tmem_ld32(tb + c0, v);
          if (lane < CW) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float f = v[e] + bv;
              if (a.relu) f = f > 0.f ? f : 0.f;
              reinterpret_cast<__nv_bfloat16*>(stg)[e * CW + lane] = __float2bfloat16_rn(f);
            }
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < PIECES; ++i) {
            const int j = lane + 32 * i;
            const int e = j / PIECES, part = j % PIECES;
            const int c = c0 + e;
            const int r = c / a.Wb;
            const int col = c - r * a.Wb;
            const int oh = oh0 + r;
            if (r < a.To_h && oh < a.Ho && col < a.Wo && nw + part * 8 < a.Og) {
              const uint4 val = *reinterpret_cast<const uint4*>(stg + e * (CW * 2) + part * 16);
              *reinterpret_cast<uint4*>(
                  out + ((static_cast<long long>(b) * a.Ho + oh) * a.Wo + col) * a.ld_out + cg0 +
                  part * 8) = val;
            }
          }
          __syncwarp();
        }
      } else {
#pragma unroll 1
      for (int sub = 0; sub < NSUB; ++sub) {
        const int m = sub * 128 + quarter * 32 + lane;
        const int r = m / a.Wb;
        const int col = m - r * a.Wb;
        const int oh = oh0 + r;
        const bool valid = r < a.To_h && oh < a.Ho && col < a.Wo;
        const long long row = (static_cast<long long>(b) * a.Ho + oh) * a.Wo + col;
        const uint32_t tb = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            acc * NSUB * BN + sub * BN;
        // 8 output channels n .. n + 7 from v[0..7]: bias + ReLU or the mask
        auto emit8 = [&](const float* v, int n) {
          if (n >= a.Og) return;
          const long long cg = static_cast<long long>(g) * a.col_goff + n;
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = v[i];
          if (a.epi == EPI_BF16) {
            if (a.bias) {
              // cg is a multiple of 8 and the staged bias 16-byte aligned
              const float4 b0 = *reinterpret_cast<const float4*>(sbias + cg);
              const float4 b1 = *reinterpret_cast<const float4*>(sbias + cg + 4);
              f[0] += b0.x;
              f[1] += b0.y;
              f[2] += b0.z;
              f[3] += b0.w;
              f[4] += b1.x;
              f[5] += b1.y;
              f[6] += b1.z;
              f[7] += b1.w;
            }
            if (a.relu) {
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] = f[i] > 0.f ? f[i] : 0.f;
            }
          } else {
            const uint4 mv = *reinterpret_cast<const uint4*>(a.mask + row * a.ld_mask + cg);
            float mf[8];
            unpack8_bits(mv, mf);
#pragma unroll
            for (int i = 0; i < 8; ++i) f[i] = mf[i] > 0.f ? f[i] : 0.f;
          }
          uint4 o;
          o.x = pack2(f[0], f[1]);
          o.y = pack2(f[2], f[3]);
          o.z = pack2(f[4], f[5]);
          o.w = pack2(f[6], f[7]);
          *reinterpret_cast<uint4*>(out + row * a.ld_out + cg) = o;
        };
        // 32-column loads alternating between the two warps of a quarter, or,
        // where that would leave one warp twice the columns of the other and
        // halves split into 16-column loads (BN = 96), each warp half of the
        // columns (32 then 16)
        constexpr bool kAlt = BN % 64 == 0 || (BN / 2) % 16 != 0;
        const int cbeg = kAlt ? 32 * half : half * (BN / 2);
        const int cend = kAlt ? BN : (half + 1) * (BN / 2);
        const int cstep = kAlt ? 64 : 32;
#pragma unroll 1
        for (int c0 = cbeg; c0 < cend; c0 += cstep) {
          if (c0 + 32 <= cend) {
            float v[32];
            tmem_ld32(tb + c0, v);
            if (!valid) continue;
#pragma unroll
            for (int h = 0; h < 4; ++h) emit8(v + 8 * h, n_t * BN + c0 + 8 * h);
          } else {
            float v[16];
            tmem_ld16(tb + c0, v);
            if (!valid) continue;
#pragma unroll
            for (int h = 0; h < 2; ++h) emit8(v + 8 * h, n_t * BN + c0 + 8 * h);
          }
        }
      }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + 8 * acc);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    for (int i = 0; i < 1000; ++i) __nanosleep(1000);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- weight gradient
// Item i = ((((split * groups + g) * cpt + ch) * n_tiles + n_t) * tsets + ts):
// tap pairs [ts * npairs / tsets, (ts + 1) * npairs / tsets) of input chunk
// ch, output channels n_t * BN .., over the position tiles of one split.
// Pair q covers taps 2q and 2q + 1; for an odd tap count the last pair's
// second half re-reads the box one row further on and is dropped.
template <int BN, int NPAIR>
__global__ void __launch_bounds__(kThreads, 1)
    conv_box_wgrad(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmY,
                   const __grid_constant__ BoxArgs a, int stages, int x_bytes) {
  constexpr int NB = (BN + 63) / 64;  // 64-channel blocks of dY per stage
  // two accumulator sets: the epilogue of item i drains one while the MMAs
  // of item i + 1 fill the other
  constexpr int ACC_COLS = NPAIR * BN;
  constexpr int TMEM_COLS = pow2_cols(2 * ACC_COLS);
  static_assert(2 * ACC_COLS <= 512, "two accumulator sets must fit in tensor memory");
  constexpr uint32_t IDESC = idesc_bf16(128, BN, 1, 1);
  // MMA warps: with two tap pairs per item, warp 9 + j issues pair j
  constexpr int NMW = NPAIR == 2 ? 2 : 1;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int y_block = a.rows_pad * 128;
  const int stage_bytes = x_bytes + NB * y_block;
  const uint32_t s0 = smem_u32(smem);
  uint8_t* barp = smem + stages * stage_bytes;
  const uint32_t full = smem_u32(barp);
  const uint32_t empty = full + 8 * stages;
  const uint32_t acc_full = empty + 8 * stages;
  const uint32_t acc_empty = acc_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(barp + 8 * (2 * stages + 4));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // dY rows past a tile's To_h * Wb positions stay zero: they are the tail
  // of the 16-row K steps and multiply box rows of other positions
  zero_smem(smem, stages * stage_bytes);
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(full + 8 * s, 1);
      mbar_init(empty + 8 * s, NMW);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(acc_full + 8 * q, NMW);
      mbar_init(acc_empty + 8 * q, 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  fence_proxy_async_smem();
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int items = a.tsets * a.n_tiles * a.cpt * a.groups * a.splits;
  const int ptiles = a.B * a.tiles_img;
  const int taps = a.K * a.K;
  const uint32_t x_box = static_cast<uint32_t>(a.Hb) * a.Wb * 128;
  const uint32_t y_box = static_cast<uint32_t>(a.To_h) * a.Wb * 128;

  if (warp == 8) {
    if (lane == 0) {
      tma_prefetch_desc(&tmX);
      tma_prefetch_desc(&tmY);
      RingPos r;
      bool ok = true;
      for (int i = blockIdx.x; i < items && ok; i += gridDim.x) {
        int q = i / a.tsets;
        const int n_t = q % a.n_tiles;
        q /= a.n_tiles;
        const int ch = q % a.cpt;
        q /= a.cpt;
        const int g = q % a.groups;
        const int sp = q / a.groups;
        const int p0 = sp * a.tiles_per_split;
        const int p1 = min(ptiles, p0 + a.tiles_per_split);
        for (int p = p0; p < p1; ++p, r.next(stages)) {
          const int b = p / a.tiles_img;
          const int oh0 = (p - b * a.tiles_img) * a.To_h;
          const int s = r.slot;
          if (!mbar_wait(empty + 8 * s, r.phase ^ 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = s0 + s * stage_bytes;
          mbar_arrive_expect_tx(full + 8 * s, x_box + NB * y_box);
          tma_load_4d(st, &tmX, g * a.cg_off + ch * 64, -a.pad, oh0 - a.pad, b, full + 8 * s);
#pragma unroll
          for (int j = 0; j < NB; ++j)
            tma_load_4d(st + x_bytes + j * y_block, &tmY, g * a.Og + n_t * BN + 64 * j, 0, oh0, b,
                        full + 8 * s);
        }
      }
    }
  } else if (warp == 9 || warp == 10) {
    const int mw = warp - 9;
    if (lane == 0 && mw < NMW) {
      // stage-relative descriptors plus the stage's start address: the
      // descriptor's start field is additive (16-byte units)
      const uint32_t sdesc0 = (s0 & 0x3FFFFu) >> 4;
      const uint64_t ydesc = smem_desc_sw128(static_cast<uint32_t>(x_bytes), y_block, 1024);
      const uint32_t y_lo = static_cast<uint32_t>(ydesc), y_hi = static_cast<uint32_t>(ydesc >> 32);
      const int ksteps = a.rows_pad / 16;
      RingPos r;
      uint32_t icount = 0;
      bool ok = true;
      for (int i = blockIdx.x; i < items && ok; i += gridDim.x, ++icount) {
        const int ts = i % a.tsets;
        const int q0 = ts * a.npairs / a.tsets;
        const int nq = (ts + 1) * a.npairs / a.tsets - q0;
        int q = i / a.tsets;
        q /= a.n_tiles;
        q /= a.cpt;
        const int sp = q / a.groups;
        const int p0 = sp * a.tiles_per_split;
        const int p1 = min(ptiles, p0 + a.tiles_per_split);
        const int acc = icount & 1;
        if (!mbar_wait(acc_empty + 8 * acc, ((icount >> 1) & 1) ^ 1, a.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t dacc = tmem_base + acc * ACC_COLS;
        // per pair: start row and leading offset of its A operand (the two
        // taps' shifts), relative to a stage's first byte
        uint32_t pair_lo[NPAIR];
        uint32_t pair_hi = 0;
#pragma unroll
        for (int j = 0; j < NPAIR; ++j) {
          const int ta = 2 * (q0 + (j < nq ? j : 0));
          const int tb = ta + 1;
          const int sa = (ta / a.K) * a.Wb + ta % a.K;
          const int sb = tb < taps ? (tb / a.K) * a.Wb + tb % a.K : sa + 1;
          const uint64_t pd = smem_desc_sw128(static_cast<uint32_t>(sa) * 128,
                                              static_cast<uint32_t>(sb - sa) * 128, 1024);
          pair_lo[j] = static_cast<uint32_t>(pd);
          pair_hi = static_cast<uint32_t>(pd >> 32);
        }
        for (int p = p0; p < p1; ++p, r.next(stages)) {
          const int s = r.slot;
          if (!mbar_wait(full + 8 * s, r.phase, a.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sdesc0 + s * (stage_bytes >> 4);
          const uint32_t acc0 = p > p0 ? 1u : 0u;
          const uint32_t bl = st + y_lo;
          if (NMW == 2) {
            // this warp's tap pair (none if the item has one pair only)
            if (mw < nq) {
              const uint32_t al = st + (mw ? pair_lo[NPAIR - 1] : pair_lo[0]);
              for (int k = 0; k < ksteps; k += 4)
                tc_mma_k4<128, 128>(dacc + mw * BN, al + k * 128, pair_hi, bl + k * 128, y_hi,
                                    IDESC, k == 0 ? acc0 : 1u);
            }
          } else {
#pragma unroll
            for (int j = 0; j < NPAIR; ++j) {
              if (j < nq) {
                const uint32_t al = st + pair_lo[j];
                for (int k = 0; k < ksteps; k += 4)
                  tc_mma_k4<128, 128>(dacc + j * BN, al + k * 128, pair_hi, bl + k * 128, y_hi,
                                      IDESC, k == 0 ? acc0 : 1u);
              }
            }
          }
          tc_commit(empty + 8 * s);
        }
        if (!ok) break;
        tc_commit(acc_full + 8 * acc);
      }
    }
  } else if (warp < 8) {
    uint32_t icount = 0;
    for (int i = blockIdx.x; i < items; i += gridDim.x, ++icount) {
      const int ts = i % a.tsets;
      const int q0 = ts * a.npairs / a.tsets;
      const int nq = (ts + 1) * a.npairs / a.tsets - q0;
      int q = i / a.tsets;
      const int n_t = q % a.n_tiles;
      q /= a.n_tiles;
      const int ch = q % a.cpt;
      q /= a.cpt;
      const int g = q % a.groups;
      const int sp = q / a.groups;
      const int acc = icount & 1;
      if (!mbar_wait(acc_full + 8 * acc, (icount >> 1) & 1, a.status, abort_flag)) break;
      tc_fence_after();
      const int quarter = warp & 3, half = warp >> 2;
      const int m = quarter * 32 + lane;  // row of D: half m / 64 of the pair, channel m % 64
      const int c = ch * 64 + (m & 63);
      float* base = a.part + sp * a.split_stride + g * a.group_stride;
#pragma unroll 1
      for (int j = 0; j < NPAIR; ++j) {
        if (j >= nq) break;
        const int tap = 2 * (q0 + j) + (m >> 6);
        const bool valid = tap < taps;
        const uint32_t tb =
            tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * ACC_COLS + j * BN;
#pragma unroll 1
        for (int c0 = 16 * half; c0 < BN; c0 += 32) {
          float v[16];
          tmem_ld16(tb + c0, v);
          if (!valid) continue;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int o = n_t * BN + c0 + e;
            if (o < a.Og) base[static_cast<long long>(o) * taps * a.P + tap * a.P + c] = v[e];
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty + 8 * acc);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    for (int i = 0; i < 1000; ++i) __nanosleep(1000);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- kernel table
struct Entry {
  int kind, bn, nsub;
  void* fn;
  bool attr;
  int kt = 0;  // forward kinds: 10 * K + taps per stage of an unrolled copy, 0 = generic
};
template <int BN, int NSUB, int BMN = 0, int SW = 0, int KT = 0>
void* fwd_ptr() {
  return reinterpret_cast<void*>(&conv_box_fwd<BN, NSUB, BMN, SW, KT>);
}
template <int BN, int NPAIR>
void* wgrad_ptr() {
  return reinterpret_cast<void*>(&conv_box_wgrad<BN, NPAIR>);
}
Entry g_entries[] = {
    {0, 48, 2, fwd_ptr<48, 2>(), false},    {0, 96, 2, fwd_ptr<96, 2>(), false},
    {0, 128, 2, fwd_ptr<128, 2>(), false},  {0, 192, 2, fwd_ptr<192, 2>(), false},
    {0, 256, 2, fwd_ptr<256, 2>(), false},  {0, 64, 2, fwd_ptr<64, 2>(), false},
    {2, 64, 2, fwd_ptr<64, 2, 1>(), false},  {2, 128, 2, fwd_ptr<128, 2, 1>(), false},
    {2, 192, 2, fwd_ptr<192, 2, 1>(), false}, {2, 256, 2, fwd_ptr<256, 2, 1>(), false},
    {2, 256, 1, fwd_ptr<256, 1, 1>(), false}, {2, 192, 1, fwd_ptr<192, 1, 1>(), false},
    {0, 192, 1, fwd_ptr<192, 1>(), false},    {0, 256, 1, fwd_ptr<256, 1>(), false},
    {3, 128, 2, fwd_ptr<128, 2, 0, 1>(), false}, {4, 64, 2, fwd_ptr<64, 2, 1, 1>(), false},
    {4, 128, 2, fwd_ptr<128, 2, 1, 1>(), false}, {5, 64, 2, fwd_ptr<64, 2, 1, 2>(), false},
    {1, 64, 4, wgrad_ptr<64, 4>(), false},  {1, 96, 2, wgrad_ptr<96, 2>(), false},
    {1, 128, 2, wgrad_ptr<128, 2>(), false},
    {1, 192, 1, wgrad_ptr<192, 1>(), false}, {1, 256, 1, wgrad_ptr<256, 1>(), false},
    // unrolled copies for the network's 3 x 3 layers (conv3-5, in stages of
    // three taps) with one accumulator per tile.  The two-sub-tile tiles
    // (conv1, conv2, conv5's forward) stay generic: unrolled, their
    // alternating MMA pairs measured slower on B200 (conv2 forward 75 ->
    // 95 us, conv5 33 -> 35 us), where these gain 5-10%.
    {3, 128, 2, fwd_ptr<128, 2, 0, 1, 33>(), false, 33},
    {4, 128, 2, fwd_ptr<128, 2, 1, 1, 33>(), false, 33},
    {0, 192, 1, fwd_ptr<192, 1, 0, 0, 33>(), false, 33},
    {2, 192, 1, fwd_ptr<192, 1, 1, 0, 33>(), false, 33},
};

Entry* find_entry(int kind, int bn, int nsub, int kt = 0) {
  for (auto& e : g_entries)
    if (e.kind == kind && e.bn == bn && e.nsub == nsub && e.kt == kt) return &e;
  return nullptr;
}

// One 128-row sub-tile per tile when two would not leave room for a second
// accumulator set in the 512 TMEM columns (N = 192, 256): the epilogue then
// still overlaps the next tile's MMAs.  Needs a box row of at most 128.
bool single_sub(int bn, const ConvShape& cs) {
  return (bn == 192 || bn == 256) && cs.Wo() + cs.K - 1 <= 128;
}

// Per FLOP, a 128 x 192 MMA reads 17% fewer operand bytes from shared
// memory than a 128 x 128 one (and one sub-tile of N = 192 keeps its
// accumulators double-buffered), so 384 outputs take two N = 192 tiles
// rather than three of 128.
int fwd_bn(int og) {
  if (og == 48 || og == 64 || og == 96 || og == 192) return og;
  if (og % 384 == 0) return 192;
  if (og % 128 == 0) return 128;
  if (og % 192 == 0) return 192;
  if (og <= 256 && og % 16 == 0) return og <= 64 ? 64 : (og <= 128 ? 128 : 256);
  return 0;
}

}  // namespace

// Shared geometry of the forward-type launches (kind 0 and 2).
static bool box_fwd_common(BoxDesc* d, const ConvShape& cs, int kind, int bn, int nsub,
                           const float* bias, int relu, const void* mask, void* y, int num_sms,
                           int* status);

bool box_desc_fwd(BoxDesc* d, const ConvShape& cs, const void* x, const void* w,
                  const float* bias, int relu, const void* mask, void* y, int num_sms,
                  int* status, bool dry) {
  memset(d, 0, sizeof(*d));
  if (cs.Cg % 8 || cs.Og % 8 || cs.C % 8 || cs.Ho() < 1 || cs.Wo() < 1) return false;
  if (bias && cs.groups * cs.Og > kMaxBias) return false;  // the bias is staged in shared memory
  int bn = fwd_bn(cs.Og);
  int nsub = single_sub(bn, cs) ? 1 : 2;
  if (!bn || !find_entry(0, bn, nsub)) return false;
  // a multiple of 128 output channels per group whose usual tile would be a
  // single 128 x 192 or 128 x 256 sub-tile (maps at most 128 - K + 1 wide,
  // conv3): the swapped tile, one 128-channel x (up to) 256-position MMA
  // per K step.  Where the usual tile has two sub-tiles, their alternating
  // accumulators issue as fast as the swapped MMA (measured, conv2 and
  // conv5) and the usual epilogue is cheaper, so it stays.
  int kind = 0;
  if (!mask && nsub == 1 && cs.Og % 128 == 0) {
    kind = 3;
    bn = 128;
    nsub = 2;
  }
  if (!box_fwd_common(d, cs, kind, bn, nsub, bias, relu, mask, y, num_sms, status)) return false;
  if (!dry) {
    const BoxArgs& a = d->args;
    if (!make_tmap_bf16_4d(&d->tmX, x, cs.C, cs.W, cs.H, cs.B, 64, a.Wb, a.Hb)) return false;
    const int Kd = cs.Kdim();
    if (!make_tmap_bf16(&d->tmW, w, Kd, static_cast<uint64_t>(cs.groups) * cs.Og,
                        static_cast<uint64_t>(Kd) * 2, 64, bn))
      return false;
  }
  return true;
}

bool box_desc_dgrad(BoxDesc* d, const ConvShape& cs, const void* dy, const void* w_fwd,
                    int p_fwd, const void* mask, void* dx, int num_sms, int* status, bool dry) {
  memset(d, 0, sizeof(*d));
  if (cs.Cg % 64 || cs.Og % 8 || cs.C % 8 || cs.Ho() < 1 || cs.Wo() < 1 || p_fwd < cs.Og)
    return false;
  // 256 output channels: one 128-row sub-tile of N = 256 (half the MMA
  // instructions of two N = 128 tiles, accumulators still double-buffered)
  int bn = cs.Og <= 64 ? 64 : (cs.Og == 192 ? 192 : (cs.Og % 128 == 0 ? 128 : 256));
  if (cs.Og % 256 == 0 && cs.Wo() + cs.K - 1 <= 128) bn = 256;
  int nsub = single_sub(bn, cs) ? 1 : 2;
  if (!find_entry(2, bn, nsub)) return false;
  // no mask and at most 64 input channels per group (conv2's 48) or a
  // multiple of 128: the swapped tile, one 64- or 128-channel x (up to)
  // 256-position MMA per K step (the MN-major weight slab as A) instead of
  // 128-position ones that need two MMAs, or leave most of the tensor pipe
  // idle with N = 64
  int kind = 2;
  if (!mask && (cs.Og <= 64 || cs.Og % 128 == 0)) {
    kind = 4;
    bn = cs.Og <= 64 ? 64 : 128;
    nsub = 2;
  }
  // at most 64 channels and a kernel of two taps or more: the tap-pair tile
  // (two taps of a kernel row on M = 128 instead of one tap on M = 64, which
  // costs the tensor pipe as much), where its stages fit
  bool done = false;
  if (kind == 4 && bn == 64 && cs.K >= 2)
    done = box_fwd_common(d, cs, 5, 64, 2, nullptr, 0, mask, dx, num_sms, status);
  if (!done &&
      !box_fwd_common(d, cs, kind, bn, nsub, nullptr, 0, mask, dx, num_sms, status))
    return false;
  d->args.w_og = cs.Cg;
  d->args.w_p = p_fwd;
  if (!dry) {
    const BoxArgs& a = d->args;
    if (!make_tmap_bf16_4d(&d->tmX, dy, cs.C, cs.W, cs.H, cs.B, 64, a.Wb, a.Hb)) return false;
    const int Kd_fwd = cs.K * cs.K * p_fwd;
    if (!make_tmap_bf16(&d->tmW, w_fwd, Kd_fwd, static_cast<uint64_t>(cs.groups) * cs.Cg,
                        static_cast<uint64_t>(Kd_fwd) * 2, 64, 64))
      return false;
  }
  return true;
}

static bool box_fwd_common(BoxDesc* d, const ConvShape& cs, int kind, int bn, int nsub,
                           const float* bias, int relu, const void* mask, void* y, int num_sms,
                           int* status) {
  BoxArgs& a = d->args;
  a.B = cs.B;
  a.Ho = cs.Ho();
  a.Wo = cs.Wo();
  a.K = cs.K;
  a.pad = cs.pad;
  a.Wb = a.Wo + cs.K - 1;
  if (a.Wb > 256) return false;
  a.To_h = (nsub * 128) / a.Wb;
  if (a.To_h < 1) return false;
  if (a.To_h > a.Ho) a.To_h = a.Ho;
  a.tiles_img = (a.Ho + a.To_h - 1) / a.To_h;
  // swapped tiles multiply only the tile's positions, rounded up to 16 (N of
  // an M = 64 or 128 MMA): 208 of the 256 for a whole 13 x 15 box
  a.sw_n = (a.To_h * a.Wb + 15) / 16 * 16;
  if (a.sw_n > 256) a.sw_n = 256;
  // rows the MMAs read: the last sub-tile's 128 rows (a swapped tile's sw_n
  // rows) at the largest shift
  const bool swapped = kind == 3 || kind == 4 || kind == 5;
  const int rows = (swapped ? a.sw_n : nsub * 128) + (cs.K - 1) * (a.Wb + 1);
  a.Hb = (rows + a.Wb - 1) / a.Wb;
  if (a.Hb > 256) return false;
  a.cpt = cs.P() / 64;
  {
    // K steps of 16 channels of the last chunk that can hold real channels;
    // only 3 (48 channels) is used to skip work, other counts run all 4
    const int real = cs.Cg - 64 * (a.cpt - 1);
    a.k16_last = (real + 15) / 16 == 3 ? 3 : 4;
  }
  a.cg_off = cs.Cg;
  a.groups = cs.groups;
  a.Og = cs.Og;
  a.n_tiles = (cs.Og + bn - 1) / bn;
  a.epi = mask ? EPI_BF16_MASK : EPI_BF16;
  a.relu = relu;
  a.out = y;
  a.ld_out = static_cast<long long>(cs.groups) * cs.Og;
  a.col_goff = cs.Og;
  a.bias = bias;
  a.mask = static_cast<const __nv_bfloat16*>(mask);
  a.ld_mask = a.ld_out;
  a.status = status;
  d->kind = kind;
  d->bn = bn;
  d->nsub = nsub;
  d->a_bytes = ((a.Hb * a.Wb * 128) + 1023) / 1024 * 1024;
  d->b_bytes = bn * 128;
  d->stages_a = 2;
  const int stg = swapped ? kStageBytes : 0;
  const int left = kSmemBudget - 1024 - kBarBytes - stg - 2 * d->a_bytes;
  // As few weight stages per input chunk as two stages in flight allow: each
  // stage costs the MMA warp a fixed ~400 clocks of hand-over beside its
  // MMAs (measured on B200: conv3's forward loop 83k / 65k / 57k clocks at
  // one / two / three taps per stage), more than a deeper ring gains.  The
  // taps are spread evenly over the stages (9 taps: 3 + 3 + 3, not 4 + 4 + 1).
  const int taps = cs.K * cs.K;
  // slabs per weight stage: the taps, or for a tap-pair tile one kernel row
  // padded to an even count (the pad slab stays zero)
  int slabs;
  if (kind == 5) {
    d->tps = cs.K;
    slabs = (cs.K + 1) & ~1;
  } else {
    int tmax = left / (2 * d->b_bytes);
    if (tmax < 1) return false;
    if (tmax > taps) tmax = taps;
    const int nst = (taps + tmax - 1) / tmax;
    d->tps = (taps + nst - 1) / nst;
    slabs = d->tps;
  }
  d->stages_b = left / (slabs * d->b_bytes);
  if (d->stages_b > 8) d->stages_b = 8;
  if (d->stages_b < 2) return false;
  d->smem = 1024 + kBarBytes + stg + 2 * d->a_bytes + d->stages_b * slabs * d->b_bytes;
  const long long tiles = 1LL * a.n_tiles * a.tiles_img * a.B * a.groups;
  d->grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  return true;
}

bool box_desc_wgrad(BoxDesc* d, const ConvShape& cs, const void* x, const void* dy,
                    float* part, int splits, int num_sms, int* status, bool dry) {
  memset(d, 0, sizeof(*d));
  if (cs.Cg % 8 || cs.Og % 8 || cs.C % 8 || cs.Ho() < 1 || cs.Wo() < 1) return false;
  BoxArgs& a = d->args;
  a.B = cs.B;
  a.Ho = cs.Ho();
  a.Wo = cs.Wo();
  a.K = cs.K;
  a.pad = cs.pad;
  a.Wb = a.Wo + cs.K - 1;
  if (a.Wb > 128) return false;
  // position tiles of at most 128 positions (8 K steps)
  a.To_h = 128 / a.Wb;
  if (a.To_h > a.Ho) a.To_h = a.Ho;
  a.rows_pad = (a.To_h * a.Wb + 63) / 64 * 64;  // whole groups of four 16-row K steps
  const int taps = cs.K * cs.K;
  // rows read: the largest second-half shift plus one (the dropped half of an
  // odd last pair) plus the K rows
  const int rows = (cs.K - 1) * (a.Wb + 1) + 1 + a.rows_pad;
  a.Hb = (rows + a.Wb - 1) / a.Wb;
  if (a.Hb > 256) return false;
  a.tiles_img = (a.Ho + a.To_h - 1) / a.To_h;
  a.cpt = cs.P() / 64;
  a.cg_off = cs.Cg;
  a.groups = cs.groups;
  a.Og = cs.Og;
  a.npairs = (taps + 1) / 2;
  a.P = cs.P();
  // output-channel tile N (the dY operand is MN-major in 64-channel blocks;
  // N = 96 reads two blocks and multiplies 96 channels of them) and pairs per
  // item within the 512 tensor-memory columns
  int bn;
  if (cs.Og <= 64)
    bn = 64;
  else if (cs.Og == 96)
    bn = 96;
  else if (cs.Og == 192)
    bn = 96;  // two tap pairs per item, one MMA warp each
  else if (cs.Og <= 128 || cs.Og % 128 == 0)
    bn = 128;
  else
    bn = 256;
  const int npair = 256 / bn;  // pairs per item: two accumulator sets of npair * bn columns
  if (!find_entry(1, bn, npair)) return false;
  a.tsets = (a.npairs + npair - 1) / npair;
  a.n_tiles = (cs.Og + bn - 1) / bn;
  const int ptiles = a.B * a.tiles_img;
  const long long base_items = 1LL * a.tsets * a.n_tiles * a.cpt * a.groups;
  if (splits <= 0) {
    // the fewest position splits that give (nearly) every SM an item and
    // fill whole waves (a mostly empty last wave costs a full item's time);
    // fewer splits also mean fewer partial sums to write and reduce
    const long long smax = ptiles / 4 > 0 ? ptiles / 4 : 1;
    long long best = 1;
    double best_eff = -1.0;
    for (long long s = 1; s <= smax && s * base_items <= 4LL * num_sms; ++s) {
      const long long items = s * base_items;
      const long long waves = (items + num_sms - 1) / num_sms;
      const double eff = static_cast<double>(items) / static_cast<double>(waves * num_sms);
      if (eff >= 0.95) {
        best = s;
        break;
      }
      if (eff > best_eff + 1e-9) {
        best_eff = eff;
        best = s;
      }
    }
    splits = static_cast<int>(best);
  }
  if (splits > ptiles) splits = ptiles;
  a.tiles_per_split = (ptiles + splits - 1) / splits;
  a.splits = (ptiles + a.tiles_per_split - 1) / a.tiles_per_split;
  a.group_stride = static_cast<long long>(cs.Og) * taps * a.P;
  a.split_stride = a.group_stride * cs.groups;
  a.part = part;
  a.status = status;
  d->kind = 1;
  d->bn = bn;
  d->nsub = npair;
  d->a_bytes = ((a.Hb * a.Wb * 128) + 1023) / 1024 * 1024;
  d->b_bytes = ((bn + 63) / 64) * a.rows_pad * 128;
  const int stage = d->a_bytes + d->b_bytes;
  int st = (kSmemBudget - 1024 - kBarBytes) / stage;
  if (st > 6) st = 6;
  if (st < 2) return false;
  d->stages_a = st;
  d->smem = 1024 + kBarBytes + st * stage;
  const long long items = base_items * a.splits;
  d->grid = static_cast<int>(items < num_sms ? items : num_sms);
  if (!dry) {
    if (!make_tmap_bf16_4d(&d->tmX, x, cs.C, cs.W, cs.H, cs.B, 64, a.Wb, a.Hb)) return false;
    if (!make_tmap_bf16_4d(&d->tmW, dy, cs.groups * cs.Og, a.Wo, a.Ho, cs.B, 64, a.Wb, a.To_h))
      return false;
  }
  return true;
}

cudaError_t box_prepare() {
  for (auto& e : g_entries) {
    if (e.attr) continue;
    cudaError_t r =
        cudaFuncSetAttribute(e.fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (r != cudaSuccess) return r;
    e.attr = true;
  }
  return cudaSuccess;
}

cudaError_t box_launch(const BoxDesc& d, cudaStream_t stream) {
  Entry* e = nullptr;
  if (d.kind != 1 && d.tps >= 1 && d.tps <= 9 && (d.args.K == 3 || d.args.K == 5))
    e = find_entry(d.kind, d.bn, d.nsub, 10 * d.args.K + d.tps);
  if (!e) e = find_entry(d.kind, d.bn, d.nsub);
  if (!e) return cudaErrorInvalidValue;
  if (!e->attr) {
    cudaError_t r =
        cudaFuncSetAttribute(e->fn, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudget);
    if (r != cudaSuccess) return r;
    e->attr = true;
  }
  count_launch();
  if (d.kind != 1) {
    void* params[] = {const_cast<CUtensorMap*>(&d.tmX), const_cast<CUtensorMap*>(&d.tmW),
                      const_cast<BoxArgs*>(&d.args), const_cast<int*>(&d.stages_a),
                      const_cast<int*>(&d.stages_b), const_cast<int*>(&d.a_bytes),
                      const_cast<int*>(&d.tps)};
    return cudaLaunchKernel(e->fn, dim3(d.grid), dim3(kThreads), params, d.smem, stream);
  }
  void* params[] = {const_cast<CUtensorMap*>(&d.tmX), const_cast<CUtensorMap*>(&d.tmW),
                    const_cast<BoxArgs*>(&d.args), const_cast<int*>(&d.stages_a),
                    const_cast<int*>(&d.a_bytes)};
  return cudaLaunchKernel(e->fn, dim3(d.grid), dim3(kThreads), params, d.smem, stream);
}

}  // namespace alx
