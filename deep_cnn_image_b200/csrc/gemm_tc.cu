// gemm_tc.cu -- the one tensor-core GEMM kernel behind every convolution and
// fully-connected product of the network (forward, data and weight gradients).
//
// Design (sm_100a):
//   * persistent: one 320-thread CTA per SM walks a static list of output
//     tiles (128 x BN), split-K slices and groups;
//   * warp roles: warps 0-7 epilogue (TMEM -> registers -> global; warps w
//     and w + 4 share TMEM lane quarter w and split the 16-column chunks
//     between them), warp 8 TMA producer, warp 9 MMA issuer (one thread)
//     and TMEM owner;
//   * operands staged in a ring of shared-memory stages laid out in the
//     128-byte-swizzled canonical form that both TMA and tcgen05.mma use;
//     full/empty mbarriers between producers and the MMA thread;
//   * two fp32 accumulators in tensor memory so the epilogue of tile i
//     overlaps the main loop of tile i+1.
// The operation itself is the plain sum D = sum_k A[m,k] B[n,k]: the
// convolution as an implicit GEMM over the (kh, kw, cin) taps
// ("ImageNet Classification with Deep Convolutional Neural Networks",
// summary page, 3.4 "Overall Architecture"; "AlexNet and Deep CNNs",
// "Time complexity of one forward pass").
#include <cudaTypedefs.h>

#include <cstdio>

#include "gemm.h"
#include "kernels.h"
#include "ptx.cuh"

namespace alx {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int NUM_THREADS = 320;
constexpr int A_TILE_BYTES = BM * BK * 2;
constexpr int MN_BLOCK_BYTES = 64 * 128;  // 64 K-rows x 64 MN elements (bf16)
// EPI_SGD_T: per epilogue warp, SGD_NBUF chunks of 16 columns x 32 rows of
// the fp32 weights and momenta staged in shared memory by cp.async
constexpr int SGD_NBUF = 3;
constexpr int SGD_CHUNK_FLOATS = 16 * 32;
constexpr int SGD_STAGE_BYTES = 8 * SGD_NBUF * 2 * SGD_CHUNK_FLOATS * 4;  // 96 KB

__host__ __device__ constexpr int tmem_cols_for(int bn) {
  return 2 * bn <= 32 ? 32 : (2 * bn <= 64 ? 64 : (2 * bn <= 128 ? 128 : (2 * bn <= 256 ? 256 : 512)));
}

struct TileCoord {
  int m_t, n_t, sp, g;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmArgs& a, int t) {
  TileCoord c;
  c.n_t = t % a.n_tiles;
  t /= a.n_tiles;
  c.m_t = t % a.m_tiles;
  t /= a.m_tiles;
  c.sp = t % a.splits;
  c.g = t / a.splits;
  return c;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN>
__device__ __forceinline__ void epilogue_store(const GemmArgs& a, const TileCoord& tc, int row,
                                               int col0, const float (&v)[16]) {
  if (row >= a.M) return;
  const int g = tc.g;
  if (a.epi == EPI_BF16 || a.epi == EPI_BF16_MASK) {
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int col = col0 + 8 * h;
      if (col >= a.N) continue;
      float f[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) f[i] = v[8 * h + i];
      const long long cg = static_cast<long long>(g) * a.col_goff + col;
      if (a.epi == EPI_BF16) {
        if (a.bias) {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] += a.bias[cg + i];
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
      o.x = pack_bf16x2(f[0], f[1]);
      o.y = pack_bf16x2(f[2], f[3]);
      o.z = pack_bf16x2(f[4], f[5]);
      o.w = pack_bf16x2(f[6], f[7]);
      *reinterpret_cast<uint4*>(out + row * a.ld_out + cg) = o;
    }
  } else if (a.epi == EPI_F32) {
    float* out = reinterpret_cast<float*>(a.out) + tc.sp * a.split_stride + g * a.group_stride +
                 row * a.ld_out;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int col = col0 + 4 * q;
      if (col < a.N)
        *reinterpret_cast<float4*>(out + col) =
            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
  } else {  // EPI_F32_T
    float* out = reinterpret_cast<float*>(a.out) + tc.sp * a.split_stride + g * a.group_stride;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int col = col0 + i;
      if (col < a.N) out[col * a.ld_out + row] = v[i];
    }
  }
}

// EPI_SGD_T: [S] 3.4 "Training Procedure Details" update rule (sgd_one)
// applied in the epilogue to the parameters whose gradients the tile holds
// (rows = input features, columns = output units of an [Out][In] matrix);
// see the epilogue below for the staging of w and v.

template <int BN, int ASRC, int BSRC>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs args, int stages) {
  constexpr int B_TILE_BYTES = BN * BK * 2;
  constexpr int TMEM_COLS = tmem_cols_for(BN);
  constexpr int A_MN = (ASRC == A_TMA_MN || ASRC == A_IM2COL_MN) ? 1 : 0;
  constexpr int B_MN = (BSRC == B_TMA_MN) ? 1 : 0;
  // the in-place update epilogue exists in the FC weight-gradient kernels only
  constexpr bool kSgd = ASRC == A_TMA_MN && BSRC == B_TMA_MN && BN % 64 == 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + stages * A_TILE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + stages * (A_TILE_BYTES + B_TILE_BYTES));
  const uint32_t bar_full = smem_u32(bars);
  const uint32_t bar_empty = bar_full + 8 * stages;
  const uint32_t bar_acc_full = bar_full + 16 * stages;
  const uint32_t bar_acc_empty = bar_acc_full + 16;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * stages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // EPI_SGD_T staging, after the barriers (whose region is under 256 bytes)
  uint8_t* sgd_stage = smem + stages * (A_TILE_BYTES + B_TILE_BYTES) + 256;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc_full + 8 * i, 1);
      mbar_init(bar_acc_empty + 8 * i, 256);
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total_tiles = args.m_tiles * args.n_tiles * args.splits * args.groups;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
      RingPos r;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
        const TileCoord tc = decode_tile(args, t);
        const int kb0 = tc.sp * args.kb_per_split;
        const int kb1 = min(args.Kblocks, kb0 + args.kb_per_split);
        // im2col, K-major: the tile's first output pixel (n, oh, ow) -> the
        // top-left input corner of its filter window
        int iw0 = 0, ih0 = 0, in0 = 0;
        if (ASRC == A_IM2COL_K) {
          const GatherDesc& G = args.g;
          const int m0 = tc.m_t * BM;
          const int HoWo = G.Ho * G.Wo;
          in0 = m0 / HoWo;
          const int rem = m0 - in0 * HoWo;
          ih0 = rem / G.Wo - G.pad;
          iw0 = rem - (rem / G.Wo) * G.Wo - G.pad;
        }
        for (int kb = kb0; kb < kb1; ++kb, r.next(stages)) {
          const int s = r.slot;
          const uint32_t ph = r.phase;
          if (!mbar_wait(bar_empty + 8 * s, ph ^ 1, args.status, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar_full + 8 * s;
          mbar_arrive_expect_tx(fb, B_TILE_BYTES + A_TILE_BYTES);
          const uint32_t dB = sB + s * B_TILE_BYTES;
          const int n0 = tc.g * args.b_goff + tc.n_t * BN;
          if (BSRC == B_TMA_K) {
            tma_load_2d(dB, &tmB, kb * BK, n0, fb);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) tma_load_2d(dB + j * MN_BLOCK_BYTES, &tmB, n0 + j * 64, kb * BK, fb);
          }
          const uint32_t dA = sA + s * A_TILE_BYTES;
          const int m0 = tc.g * args.a_goff + tc.m_t * BM;
          if (ASRC == A_TMA_K) {
            tma_load_2d(dA, &tmA, kb * BK, m0, fb);
          } else if (ASRC == A_TMA_MN) {
            tma_load_2d(dA, &tmA, m0, kb * BK, fb);
            tma_load_2d(dA + MN_BLOCK_BYTES, &tmA, m0 + 64, kb * BK, fb);
          } else if (ASRC == A_IM2COL_K) {
            // k-block kb = (tap, 64-channel chunk)
            const GatherDesc& G = args.g;
            const int tap = kb / G.cpt;
            const int chunk = kb - tap * G.cpt;
            const int kh = tap / G.KW, kw = tap - (tap / G.KW) * G.KW;
            tma_load_im2col_4d(dA, &tmA, tc.g * G.cg_off + chunk * 64, iw0, ih0, in0,
                               static_cast<uint16_t>(kw), static_cast<uint16_t>(kh), fb);
          } else if (ASRC == A_IM2COL_MN) {
            // k-block kb = 64 output pixels (the reduction); the tile's two
            // 64-wide M blocks are (tap, 64-channel chunk) pairs
            const GatherDesc& G = args.g;
            const int p0 = kb * BK;
            const int HoWo = G.Ho * G.Wo;
            const int n = p0 / HoWo;
            const int rem = p0 - n * HoWo;
            const int oh = rem / G.Wo, ow = rem - (rem / G.Wo) * G.Wo;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              // blocks past the last tap (the M tail) load tap 0; their rows
              // are never stored
              const int mb = min(tc.m_t * 2 + j, G.Kc - 1) * (tc.m_t * 2 + j < G.Kc);
              const int tap = mb / G.cpt;
              const int chunk = mb - tap * G.cpt;
              const int kh = tap / G.KW, kw = tap - (tap / G.KW) * G.KW;
              tma_load_im2col_4d(dA + j * MN_BLOCK_BYTES, &tmA, tc.g * G.cg_off + chunk * 64,
                                 ow - G.pad, oh - G.pad, n, static_cast<uint16_t>(kw),
                                 static_cast<uint16_t>(kh), fb);
            }
          }
        }
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, BN, A_MN, B_MN);
      const uint64_t adesc0 = A_MN ? smem_desc_sw128(sA, MN_BLOCK_BYTES, 1024)
                                   : smem_desc_sw128(sA, 16, 1024);
      const uint64_t bdesc0 = B_MN ? smem_desc_sw128(sB, MN_BLOCK_BYTES, 1024)
                                   : smem_desc_sw128(sB, 16, 1024);
      const uint32_t a_lo0 = static_cast<uint32_t>(adesc0), a_hi = static_cast<uint32_t>(adesc0 >> 32);
      const uint32_t b_lo0 = static_cast<uint32_t>(bdesc0), b_hi = static_cast<uint32_t>(bdesc0 >> 32);
      RingPos r;
      uint32_t tcount = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tcount) {
        const TileCoord tc = decode_tile(args, t);
        const int kb0 = tc.sp * args.kb_per_split;
        const int kb1 = min(args.Kblocks, kb0 + args.kb_per_split);
        const int acc = tcount & 1;
        const uint32_t aph = (tcount >> 1) & 1;
        if (!mbar_wait(bar_acc_empty + 8 * acc, aph ^ 1, args.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * (TMEM_COLS / 2);
        for (int kb = kb0; kb < kb1; ++kb, r.next(stages)) {
          const int s = r.slot;
          const uint32_t ph = r.phase;
          if (!mbar_wait(bar_full + 8 * s, ph, args.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptors advance by adding 16-byte units to the start field
          tc_mma_k4<A_MN ? 128 : 2, B_MN ? 128 : 2>(
              d_tmem, a_lo0 + s * (A_TILE_BYTES >> 4), a_hi, b_lo0 + s * (B_TILE_BYTES >> 4), b_hi,
              idesc, kb == kb0 ? 0u : 1u);
          tc_commit(bar_empty + 8 * s);
        }
        if (!ok) break;
        tc_commit(bar_acc_full + 8 * acc);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    uint32_t tcount = 0;
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int row_in_tile = quarter * 32 + lane;
    HParams hp{};
    if (kSgd && args.epi == EPI_SGD_T) hp = *args.hp;
    for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++tcount) {
      const TileCoord tc = decode_tile(args, t);
      const int acc = tcount & 1;
      const uint32_t aph = (tcount >> 1) & 1;
      if (!mbar_wait(bar_acc_full + 8 * acc, aph, args.status, abort_flag)) break;
      tc_fence_after();
      const int row = tc.m_t * BM + row_in_tile;
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * (TMEM_COLS / 2);
      if (kSgd && args.epi == EPI_SGD_T) {
        // each half of the warps takes a contiguous half of the columns, in
        // chunks of 16; a chunk's w and v (16 lines of 128 bytes each: the 32
        // rows of this warp) arrive in shared memory by cp.async SGD_NBUF - 1
        // chunks ahead, so many lines are in flight without holding registers
        const int cb = half * (BN / 2);
        constexpr int nchunks = BN / 2 / 16;
        const int row_base = tc.m_t * BM + quarter * 32;
        const size_t ld = static_cast<size_t>(args.ld_out);
        float* sw = reinterpret_cast<float*>(sgd_stage) + warp * (SGD_NBUF * 2 * SGD_CHUNK_FLOATS);
        auto issue = [&](int c) {
          const int buf = c % SGD_NBUF;
          float* dw = sw + buf * 2 * SGD_CHUNK_FLOATS;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int pidx = lane + 32 * t;
            const int col = pidx >> 3, part = pidx & 7;
            const int o = tc.n_t * BN + cb + 16 * c + col;
            if (o < args.N && row_base < args.M) {  // M % 32 == 0: all 32 rows exist
              const size_t src = static_cast<size_t>(o) * ld + row_base + part * 4;
              cp_async16(smem_u32(dw + col * 32 + part * 4), args.sgd_w + src);
              cp_async16(smem_u32(dw + SGD_CHUNK_FLOATS + col * 32 + part * 4), args.sgd_v + src);
            }
          }
          cp_async_commit();
        };
        const bool live = row < args.M;
#pragma unroll 1
        for (int c = 0; c < nchunks; ++c) {
          if (c == 0) {
#pragma unroll
            for (int q = 0; q < SGD_NBUF - 1; ++q) {
              if (q < nchunks) issue(q);
              else cp_async_commit();
            }
          }
          if (c + SGD_NBUF - 1 < nchunks) issue(c + SGD_NBUF - 1);
          else cp_async_commit();
          cp_async_wait<SGD_NBUF - 1>();
          __syncwarp();
          const float* srcw = sw + (c % SGD_NBUF) * 2 * SGD_CHUNK_FLOATS;
          float g[16];
          tmem_ld16(tbase + cb + 16 * c, g);  // every lane takes part (warp-wide load)
          const int o0 = tc.n_t * BN + cb + 16 * c;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (live && o0 + i < args.N) {
              float wv = srcw[i * 32 + lane], vv = srcw[SGD_CHUNK_FLOATS + i * 32 + lane];
              sgd_one(wv, vv, g[i], hp);
              const size_t e = static_cast<size_t>(o0 + i) * ld + row;
              args.sgd_w[e] = wv;
              args.sgd_v[e] = vv;
              args.sgd_shadow[e] = __float2bfloat16_rn(wv);
              if (args.sgd_grads) args.sgd_grads[e] = g[i];
            }
          }
          __syncwarp();  // the buffer is refilled next
        }
      } else {
#pragma unroll 1
        for (int c0 = 16 * half; c0 < BN; c0 += 32) {
          float v[16];
          tmem_ld16(tbase + c0, v);
          epilogue_store<BN>(args, tc, row, tc.n_t * BN + c0, v);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_acc_empty + 8 * acc);
    }
  }

  __syncthreads();
  if (*abort_flag) {
    // give bulk copies already in flight time to land before the CTA exits
    for (int i = 0; i < 1000; ++i) __nanosleep(1000);
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

using KernelFn = void (*)(CUtensorMap, CUtensorMap, GemmArgs, int);

template <int BN, int ASRC, int BSRC>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&gemm_kernel<BN, ASRC, BSRC>);
}

struct KernelEntry {
  int bn, asrc, bsrc;
  void* fn;
  bool attr_set;
};

#define ALX_K(BN_, A_, B_) {BN_, A_, B_, kernel_ptr<BN_, A_, B_>(), false}
KernelEntry g_kernels[] = {
    ALX_K(64, A_TMA_K, B_TMA_K),       ALX_K(128, A_TMA_K, B_TMA_K),
    ALX_K(256, A_TMA_K, B_TMA_K),      ALX_K(64, A_TMA_K, B_TMA_MN),
    ALX_K(128, A_TMA_K, B_TMA_MN),     ALX_K(256, A_TMA_K, B_TMA_MN),
    ALX_K(64, A_TMA_MN, B_TMA_MN),     ALX_K(128, A_TMA_MN, B_TMA_MN),
    ALX_K(256, A_TMA_MN, B_TMA_MN),
    ALX_K(48, A_IM2COL_K, B_TMA_K),    ALX_K(64, A_IM2COL_K, B_TMA_K),
    ALX_K(96, A_IM2COL_K, B_TMA_K),    ALX_K(128, A_IM2COL_K, B_TMA_K),
    ALX_K(192, A_IM2COL_K, B_TMA_K),   ALX_K(256, A_IM2COL_K, B_TMA_K),
    ALX_K(64, A_IM2COL_MN, B_TMA_MN),  ALX_K(128, A_IM2COL_MN, B_TMA_MN),
    ALX_K(192, A_IM2COL_MN, B_TMA_MN), ALX_K(256, A_IM2COL_MN, B_TMA_MN),
};
#undef ALX_K

KernelEntry* find_kernel(int bn, int asrc, int bsrc) {
  for (auto& k : g_kernels)
    if (k.bn == bn && k.asrc == asrc && k.bsrc == bsrc) return &k;
  return nullptr;
}

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool load_encode() {
  if (g_encode) return true;
  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  if (!load_encode()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (row_bytes & 15) || inner == 0 || outer == 0)
    return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_bf16_4d(CUtensorMap* m, const void* base, int C, int W, int H, int N,
                       uint32_t box_c, uint32_t box_w, uint32_t box_h) {
  if (!load_encode()) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (C * 2) % 16 || C < 1 || W < 1 || H < 1 ||
      N < 1 || box_c * 2 > 128 || box_w > 256 || box_h > 256)
    return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(W) * C * 2,
                           static_cast<cuuint64_t>(H) * W * C * 2};
  cuuint32_t box[4] = {box_c, box_w, box_h, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

namespace {
PFN_cuTensorMapEncodeIm2col_v12000 g_encode_im2col = nullptr;
}

bool make_tmap_im2col(CUtensorMap* m, const void* base, int N, int H, int W, int C, int K,
                      int pad, int pixels) {
  if (!g_encode_im2col) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeIm2col", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    g_encode_im2col = reinterpret_cast<PFN_cuTensorMapEncodeIm2col_v12000>(fn);
  }
  if ((reinterpret_cast<uintptr_t>(base) & 15) || (C * 2) % 16 || N < 1 || H < 1 || W < 1)
    return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                        static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(N)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2, static_cast<cuuint64_t>(W) * C * 2,
                           static_cast<cuuint64_t>(H) * W * C * 2};
  // bounding box of the filter window's top-left corner, in (W, H) order:
  // from -pad to (size - 1) + (pad - (K - 1))
  int lower[2] = {-pad, -pad};
  int upper[2] = {pad - (K - 1), pad - (K - 1)};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode_im2col(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base),
                               dims, strides, lower, upper, 64, static_cast<cuuint32_t>(pixels),
                               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool gemm_finalize(GemmDesc* d, int num_sms) {
  KernelEntry* k = find_kernel(d->bn, d->asrc, d->bsrc);
  if (!k) return false;
  GemmArgs& a = d->args;
  if (a.M <= 0 || a.N <= 0 || a.Kblocks <= 0 || a.groups <= 0) return false;
  if (a.N % 8) return false;
  if (d->bsrc == B_TMA_MN && d->bn % 64) return false;
  if (a.epi == EPI_SGD_T &&
      (d->asrc != A_TMA_MN || d->bsrc != B_TMA_MN || d->bn % 64 || a.groups != 1 ||
       a.kb_per_split < a.Kblocks))
    return false;
  a.m_tiles = (a.M + BM - 1) / BM;
  a.n_tiles = (a.N + d->bn - 1) / d->bn;
  if (a.kb_per_split <= 0 || a.kb_per_split > a.Kblocks) a.kb_per_split = a.Kblocks;
  a.splits = (a.Kblocks + a.kb_per_split - 1) / a.kb_per_split;
  const int stage_bytes = A_TILE_BYTES + d->bn * BK * 2;
  // the in-place update stages its fp32 weights and momenta (rows in
  // 16-byte pieces: M % 32 == 0 keeps every piece inside the matrix)
  const bool sgd = a.epi == EPI_SGD_T;
  if (sgd && a.M % 32) return false;
  const int extra = sgd ? SGD_STAGE_BYTES : 0;
  const int budget = 227 * 1024 - 1024 - 256 - extra;
  int stages = budget / stage_bytes;
  if (stages > 8) stages = 8;
  if (stages < (sgd ? 2 : 3)) return false;
  d->stages = stages;
  d->smem = stages * stage_bytes + 1024 + 256 + extra;
  const long long tiles = 1LL * a.m_tiles * a.n_tiles * a.splits * a.groups;
  d->grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
  return true;
}

cudaError_t gemm_prepare() {
  for (auto& k : g_kernels) {
    if (k.attr_set) continue;
    cudaError_t e = cudaFuncSetAttribute(k.fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    k.attr_set = true;
  }
  return cudaSuccess;
}

cudaError_t gemm_launch(const GemmDesc& d, cudaStream_t stream) {
  KernelEntry* k = find_kernel(d.bn, d.asrc, d.bsrc);
  if (!k) return cudaErrorInvalidValue;
  if (!k->attr_set) {
    cudaError_t e = cudaFuncSetAttribute(k->fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e != cudaSuccess) return e;
    k->attr_set = true;
  }
  void* params[] = {const_cast<CUtensorMap*>(&d.tmA), const_cast<CUtensorMap*>(&d.tmB),
                    const_cast<GemmArgs*>(&d.args), const_cast<int*>(&d.stages)};
  count_launch();
  return cudaLaunchKernel(k->fn, dim3(d.grid), dim3(NUM_THREADS), params, d.smem, stream);
}

}  // namespace alx
