// net.cu -- the host side of libalexnet.so: handle, workspace layout,
// per-batch GEMM plans and the order of launches of a forward pass and of a
// training step.  All device memory is the caller's workspace; nothing here
// allocates device memory.
//
// Pages cited:
//   [S] "ImageNet Classification with Deep Convolutional Neural Networks",
//       paper-graph-ui summary page (section 3.4 subsections).
//   [W] "AlexNet and Deep CNNs" (fermi.ai wiki page), listings
//       ALEXNET_FORWARD and TRAIN_STEP.
#include <cstdio>
#include <cstring>
#include <map>
#include <string>
#include <vector>

#include "alexnet.h"
#include "alexnet_ops.h"
#include "conv_desc.h"
#include "gemm.h"
#include "kernels.h"

using namespace alx;

namespace {

constexpr int kClasses = 1000;

// Guard region after every workspace buffer: filled with kCanaryByte at
// create and compared by alexnet_debug_canaries, so that a kernel writing
// past the end of any buffer is caught.
constexpr size_t kCanaryBytes = 256;
constexpr unsigned char kCanaryByte = 0xA5;

// Bump allocator over the caller's workspace (base == nullptr: size only).
// Every buffer starts on a 256-byte boundary and is followed by a guard.
struct Carver {
  char* base;
  size_t off = 0;
  std::vector<size_t>* guards;  // offsets of the guard regions (nullable)
  explicit Carver(void* b, std::vector<size_t>* g = nullptr)
      : base(static_cast<char*>(b)), guards(g) {}
  template <typename T>
  T* take(size_t n) {
    off = (off + 255) & ~static_cast<size_t>(255);
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += n * sizeof(T);
    if (guards) guards->push_back(off);
    off += kCanaryBytes;
    return p;
  }
};

struct ConvL {
  int Cin, Cout, K, stride, pad, groups;
  int H, Ho;    // input / output side
  int lrn, pool;
  int P;        // side after pooling (or Ho)
  // GEMM view (conv1 is the 3x3 stride-1 convolution of its 57x57x48
  // space-to-depth input)
  int gH, gC, gK, gpad, gCg;
  int Og() const { return Cout / groups; }
  int Pch() const { return 64 * ((gCg + 63) / 64); }  // channels per tap, padded
  int Kdim() const { return gK * gK * Pch(); }
  // GEMM views: forward / weight gradient over the layer input, and the data
  // gradient as a forward convolution of dY with the flipped kernel
  ConvShape fwd(int B) const { return ConvShape{B, gH, gH, gC, gCg, Og(), groups, gK, gpad}; }
  ConvShape dgrad(int B) const {
    return ConvShape{B, Ho, Ho, Cout, Og(), Cin / groups, groups, K, K - 1 - pad};
  }
};

struct FcL {
  int In, Out;
};

struct Plan {
  ConvPlan cf[5], cd[5], cw[5];
  GemmDesc ff[3], fd[3], fw[3];
  GemmDesc fws[3];  // FC weight gradient with the update in its epilogue
  GemmDesc fwg[3];  // FC weight gradient straight into the handle's gradient buffer
  bool has_fwg = false;
  double conv_flops[5], fc_flops[3];  // algorithmic FLOPs of one pass of each layer
  bool ok = false;
};

// K blocks per split of a split-K GEMM with `tiles` output tiles: the split
// count that minimises waves x (K blocks per item + a fixed per-item cost of
// writing its fp32 partial tile, about two K blocks of loads), preferring
// fewer splits (fewer partials to reduce) on ties.
int pick_kbps(long long tiles, int kblocks, int num_sms, int min_blocks) {
  const int smax = kblocks / min_blocks > 0 ? kblocks / min_blocks : 1;
  int best_kbps = kblocks;
  long long best_cost = -1;
  for (int s = 1; s <= smax; ++s) {
    const int kbps = (kblocks + s - 1) / s;
    const long long items = tiles * ((kblocks + kbps - 1) / kbps);
    const long long waves = (items + num_sms - 1) / num_sms;
    const long long cost = waves * (kbps + 2);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_kbps = kbps;
    }
  }
  return best_kbps;
}

}  // namespace

struct alexnet {
  alexnet_config cfg;
  int num_sms = 148;
  char* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<size_t> guards;  // workspace offsets of the guard regions
  std::string err;
  cudaStream_t last_stream = nullptr;
  uint64_t step = 0;

  ConvL conv[5];
  FcL fc[3];
  size_t w_off[8], w_len[8], b_off[8], b_len[8];
  size_t n_params = 0;

  // device buffers
  float* params = nullptr;  // [n_params] then vel [n_params] contiguous
  float* vel = nullptr;
  float* grads = nullptr;
  bf16* wf[8] = {};  // forward GEMM operands
  bf16* wd[5] = {};  // data-gradient operands (conv2..conv5)
  HParams* hp = nullptr;
  int* status = nullptr;
  float* loss_dev = nullptr;
  float* loss_rows = nullptr;
  bf16* xin = nullptr;  // staged inputs (ten-crop patches)
  bf16* xs = nullptr;
  bf16* a[5] = {};
  bf16* lo[5] = {};
  bf16* p[5] = {};
  uint8_t* am[5] = {};
  bf16* f6 = nullptr;
  bf16* f7 = nullptr;
  float* logits = nullptr;
  float* probs = nullptr;
  bf16* dlogits = nullptr;
  bf16* d7 = nullptr;
  bf16* d6 = nullptr;
  bf16* dp5 = nullptr;
  bf16* da[5] = {};
  bf16* dp[5] = {};
  bf16* dl[5] = {};
  float* scratch = nullptr;
  size_t scratch_floats = 0;
  float* cpart = nullptr;
  size_t cpart_floats = 0;
  size_t cpart_off[5] = {0, 0, 0, 0, 0};  // per conv layer, floats
  // fp32 path
  float* fa = nullptr;
  float* fb = nullptr;
  float* fwt = nullptr;
  size_t f_act = 0;

  HParams hp_host;
  std::map<int, Plan> plans;

  // CUDA graphs of the training step, one per batch size (see train_step)
  int32_t* labels_buf = nullptr;
  cudaStream_t cap_stream = nullptr;
  std::map<int, cudaGraphExec_t> train_graphs;
  std::map<int, int64_t> graph_kernels;  // kernels in each captured step
  bool use_graphs = true;

  // launch accounting (alexnet_stats_*): the GEMM events of one call; a
  // captured graph owns the events recorded into it (as event-record nodes)
  struct StepRec {
    std::vector<cudaEvent_t> ev;  // start/stop pairs
    size_t used = 0;
    int64_t gemm_launches = 0;
    double gemm_flops = 0.0;
    std::vector<double> flops;  // per GEMM launch, in launch order
    std::vector<int> kind;      // 0: convolution, 1: FC forward / data gradient, 2: FC weight gradient
    void reset() {
      used = 0;
      gemm_launches = 0;
      gemm_flops = 0.0;
      flops.clear();
      kind.clear();
    }
  };
  bool stats_on = false;
  // also store the normalised maps (lo) and their gradients (dl), which the
  // fused normalisation + pooling kernels otherwise keep on chip
  bool keep = false;
  // FC weights updated by the weight-gradient GEMM's epilogue (else by a
  // separate update kernel reading an fp32 gradient)
  bool fc_fused = true;
  // the flipped weight copies (wd) are refreshed only while some data-gradient
  // plan reads them (the box kernel reads the forward copies transposed)
  bool need_wd = false;
  // data-parallel gradient step (alexnet_train_grads): no update, every
  // parameter gradient written to `grads`, dropout rows offset by the first
  // image's index in the whole minibatch; fc_event marks the FC gradients
  bool grads_only = false;
  uint32_t row_offset = 0;
  cudaEvent_t fc_event = nullptr;
  // conv weight gradients and updates run on a second stream beside the
  // data-gradient chain (fork when dY is complete, the update after the
  // data gradient that reads the layer's old weights, join at the end)
  bool overlap_wgrad = true;
  cudaStream_t side = nullptr;
  cudaEvent_t ev_dy[5] = {}, ev_dg[5] = {}, ev_join = nullptr;
  cudaEvent_t ev_fdz[3] = {}, ev_fdg[3] = {}, ev_fjoin = nullptr;  // the FC layers'


  bool capturing = false;
  StepRec direct_rec;
  std::map<int, StepRec> graph_rec;
  StepRec* rec = nullptr;       // where run_gemm records
  StepRec* last_rec = nullptr;  // the most recent call's record
  int64_t last_launches = 0;
  cudaStream_t stats_stream = nullptr;

  const bf16* conv_input(int l) const {
    if (l == 0) return xs;
    const int q = l - 1;
    if (conv[q].pool) return p[q];
    if (conv[q].lrn) return lo[q];
    return a[q];
  }
};

namespace {

std::string g_create_error;

bool set_err(alexnet* h, const char* msg) {
  if (h) h->err = msg;
  return false;
}

alexnet_status cuda_status(alexnet* h, cudaError_t e, const char* where) {
  if (e == cudaSuccess) return ALEXNET_OK;
  char buf[256];
  snprintf(buf, sizeof(buf), "%s: %s", where, cudaGetErrorString(e));
  if (h) h->err = buf;
  return ALEXNET_ERR_CUDA;
}

bool valid_config(const alexnet_config* c) {
  if (!c) return false;
  if (c->batch_max < 1 || c->batch_max > 4096) return false;
  if (c->dtype != ALEXNET_FP32 && c->dtype != ALEXNET_BF16) return false;
  if (c->grouped != 0 && c->grouped != 1) return false;
  if (c->lrn_n != 5) return false;
  if (c->pool_size != 2 && c->pool_size != 3) return false;
  if (!(c->dropout_p >= 0.f && c->dropout_p < 1.f)) return false;
  if (!(c->lrn_k > 0.f)) return false;
  return true;
}

void build_geometry(alexnet* h) {
  const alexnet_config& c = h->cfg;
  const int g = c.grouped ? 2 : 1;
  const int cin[5] = {3, 96, 256, 384, 384};
  const int cout[5] = {96, 256, 384, 384, 256};
  const int ks[5] = {11, 5, 3, 3, 3};
  const int st[5] = {4, 1, 1, 1, 1};
  const int pd[5] = {0, 2, 1, 1, 1};
  const int gr[5] = {1, g, 1, g, g};
  const int lrn[5] = {c.lrn_on, c.lrn_on, 0, 0, 0};
  const int pool[5] = {1, 1, 0, 0, 1};
  int H = 227;
  size_t off = 0;
  for (int l = 0; l < 5; ++l) {
    ConvL& L = h->conv[l];
    L.Cin = cin[l];
    L.Cout = cout[l];
    L.K = ks[l];
    L.stride = st[l];
    L.pad = pd[l];
    L.groups = gr[l];
    L.H = H;
    L.Ho = (H + 2 * L.pad - L.K) / L.stride + 1;
    L.lrn = lrn[l];
    L.pool = pool[l];
    L.P = L.pool ? (L.Ho - c.pool_size) / 2 + 1 : L.Ho;
    if (l == 0) {
      L.gH = 57;
      L.gC = 64;
      L.gK = 3;
      L.gpad = 0;
      L.gCg = 48;
    } else {
      L.gH = H;
      L.gC = L.Cin;
      L.gK = L.K;
      L.gpad = L.pad;
      L.gCg = L.Cin / L.groups;
    }
    h->w_off[l] = off;
    h->w_len[l] = static_cast<size_t>(L.Cout) * L.K * L.K * (L.Cin / L.groups);
    off += h->w_len[l];
    h->b_off[l] = off;
    h->b_len[l] = L.Cout;
    off += h->b_len[l];
    H = L.P;
  }
  int in = H * H * h->conv[4].Cout;
  const int outs[3] = {4096, 4096, kClasses};
  for (int f = 0; f < 3; ++f) {
    h->fc[f].In = in;
    h->fc[f].Out = outs[f];
    h->w_off[5 + f] = off;
    h->w_len[5 + f] = static_cast<size_t>(in) * outs[f];
    off += h->w_len[5 + f];
    h->b_off[5 + f] = off;
    h->b_len[5 + f] = outs[f];
    off += h->b_len[5 + f];
    in = outs[f];
  }
  h->n_params = off;
}

// ---------------------------------------------------------------- GEMM descs
// When sizing the workspace no tensor map is encoded (no device is needed).
bool g_dry_tmaps = false;

bool tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
          uint32_t box_inner, uint32_t box_outer) {
  if (g_dry_tmaps) {
    memset(m, 0, sizeof(*m));
    return true;
  }
  return make_tmap_bf16(m, base, inner, outer, row_bytes, box_inner, box_outer);
}

bool desc_fc_fwd(GemmDesc* d, const FcL& F, const bf16* x, const bf16* w, float* part, int B,
                 int splits, int num_sms, int* status) {
  memset(d, 0, sizeof(*d));
  d->asrc = A_TMA_K;
  d->bsrc = B_TMA_K;
  d->bn = 128;
  GemmArgs& a = d->args;
  a.M = B;
  a.N = F.Out;
  a.Kblocks = (F.In + 63) / 64;
  a.groups = 1;
  const long long tiles = 1LL * ((B + 127) / 128) * ((F.Out + 127) / 128);
  a.kb_per_split = splits > 0 ? (a.Kblocks + splits - 1) / splits
                              : pick_kbps(tiles, a.Kblocks, num_sms, 4);
  a.epi = EPI_F32;
  a.out = part;
  a.ld_out = F.Out;
  a.split_stride = 1LL * B * F.Out;
  a.status = status;
  if (!tmap(&d->tmA, x, F.In, B, static_cast<uint64_t>(F.In) * 2, 64, 128)) return false;
  if (!tmap(&d->tmB, w, F.In, F.Out, static_cast<uint64_t>(F.In) * 2, 64, 128))
    return false;
  return gemm_finalize(d, num_sms);
}

bool desc_fc_dgrad(GemmDesc* d, const FcL& F, const bf16* dz, const bf16* w, float* part, int B,
                   int splits, int num_sms, int* status) {
  memset(d, 0, sizeof(*d));
  d->asrc = A_TMA_K;
  d->bsrc = B_TMA_MN;
  d->bn = F.In % 256 == 0 ? 256 : 128;
  GemmArgs& a = d->args;
  a.M = B;
  a.N = F.In;
  a.Kblocks = (F.Out + 63) / 64;
  a.groups = 1;
  const long long tiles = 1LL * ((B + 127) / 128) * ((F.In + d->bn - 1) / d->bn);
  a.kb_per_split = splits > 0 ? (a.Kblocks + splits - 1) / splits
                              : pick_kbps(tiles, a.Kblocks, num_sms, 4);
  a.epi = EPI_F32;
  a.out = part;
  a.ld_out = F.In;
  a.split_stride = 1LL * B * F.In;
  a.status = status;
  if (!tmap(&d->tmA, dz, F.Out, B, static_cast<uint64_t>(F.Out) * 2, 64, 128))
    return false;
  if (!tmap(&d->tmB, w, F.In, F.Out, static_cast<uint64_t>(F.In) * 2, 64, 64))
    return false;
  return gemm_finalize(d, num_sms);
}


// FC weight gradient dW[o][i] = sum_b dz[b][o] x[b][i], computed as
// D[i][o] (rows = input features): the epilogue's lanes are consecutive
// input features, so each column o is written as 128 contiguous bytes of
// the fp32 [out][in] gradient (to scratch, for k_sgd_dense).
bool desc_fc_wgrad(GemmDesc* d, const FcL& F, const bf16* dz, const bf16* x, float* out, int B,
                   int num_sms, int* status) {
  memset(d, 0, sizeof(*d));
  d->asrc = A_TMA_MN;
  d->bsrc = B_TMA_MN;
  d->bn = F.Out % 256 == 0 ? 256 : 128;
  GemmArgs& a = d->args;
  a.M = F.In;
  a.N = F.Out;
  a.Kblocks = (B + 63) / 64;
  a.groups = 1;
  a.kb_per_split = a.Kblocks;
  a.epi = EPI_F32_T;
  a.out = out;
  a.ld_out = F.In;
  a.split_stride = static_cast<long long>(F.In) * F.Out;
  a.group_stride = 0;
  a.status = status;
  if (!tmap(&d->tmA, x, F.In, B, static_cast<uint64_t>(F.In) * 2, 64, 64)) return false;
  if (!tmap(&d->tmB, dz, F.Out, B, static_cast<uint64_t>(F.Out) * 2, 64, 64)) return false;
  return gemm_finalize(d, num_sms);
}

// The same product with [S] 3.4's update applied by the epilogue: w, v
// ([Out][In] fp32) updated in place, the bf16 copy refreshed, the gradient
// kept in grads when given.  No fp32 gradient reaches global memory.
bool desc_fc_wgrad_sgd(GemmDesc* d, const FcL& F, const bf16* dz, const bf16* x, float* w,
                       float* v, bf16* shadow, float* grads, const HParams* hp, int B,
                       int num_sms, int* status) {
  if (!desc_fc_wgrad(d, F, dz, x, nullptr, B, num_sms, status)) return false;
  GemmArgs& a = d->args;
  a.epi = EPI_SGD_T;
  a.sgd_w = w;
  a.sgd_v = v;
  a.sgd_shadow = shadow;
  a.sgd_grads = grads;
  a.hp = hp;
  return gemm_finalize(d, num_sms);
}

size_t desc_f32_need(const GemmDesc& d) {
  const GemmArgs& a = d.args;
  if (a.epi == EPI_F32_T) return static_cast<size_t>(a.splits) * a.split_stride;
  if (a.epi == EPI_F32)
    return a.split_stride ? static_cast<size_t>(a.splits) * a.split_stride
                          : static_cast<size_t>(a.M) * a.ld_out;
  return 0;
}

bool build_plan(alexnet* h, int B, Plan* P) {
  const int ns = h->num_sms;
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    if (!conv_plan_fwd(&P->cf[l], L.fwd(B), h->conv_input(l), h->wf[l], h->params + h->b_off[l], 1,
                       nullptr, h->a[l], ns, h->status, g_dry_tmaps))
      return set_err(h, "conv forward plan");
    if (l > 0) {
      const bf16* mask = (!h->conv[l - 1].pool) ? h->a[l - 1] : nullptr;
      bf16* out = mask ? h->da[l - 1] : h->dp[l - 1];
      if (!conv_plan_dgrad(&P->cd[l], L.dgrad(B), h->da[l], h->wf[l], L.Pch(), h->wd[l], mask,
                           out, ns, h->status, g_dry_tmaps))
        return set_err(h, "conv data-gradient plan");
      if (!P->cd[l].box) h->need_wd = true;
    }
    if (!conv_plan_wgrad(&P->cw[l], L.fwd(B), h->conv_input(l), h->da[l], h->scratch, 0, ns,
                         h->status, g_dry_tmaps))
      return set_err(h, "conv weight-gradient plan");
  }
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    P->conv_flops[l] = 2.0 * B * L.Ho * L.Ho * L.Cout * L.K * L.K * (L.Cin / L.groups);
  }
  for (int f = 0; f < 3; ++f) P->fc_flops[f] = 2.0 * B * h->fc[f].In * h->fc[f].Out;
  const bf16* fin[3] = {h->p[4], h->f6, h->f7};
  const bf16* dz[3] = {h->d6, h->d7, h->dlogits};
  for (int f = 0; f < 3; ++f) {
    if (!desc_fc_fwd(&P->ff[f], h->fc[f], fin[f], h->wf[5 + f], h->scratch, B, 0, ns, h->status))
      return set_err(h, "fc forward plan");
    if (!desc_fc_dgrad(&P->fd[f], h->fc[f], dz[f], h->wf[5 + f], h->scratch, B, 0, ns, h->status))
      return set_err(h, "fc data-gradient plan");
    if (!desc_fc_wgrad(&P->fw[f], h->fc[f], dz[f], fin[f], h->scratch, B, ns, h->status))
      return set_err(h, "fc weight-gradient plan");
    float* gr = h->grads ? h->grads + h->w_off[5 + f] : nullptr;
    if (!desc_fc_wgrad_sgd(&P->fws[f], h->fc[f], dz[f], fin[f], h->params + h->w_off[5 + f],
                           h->vel + h->w_off[5 + f], h->wf[5 + f], gr, h->hp, B, ns, h->status))
      return set_err(h, "fc weight-gradient + update plan");
    // one K-slice (the batch fits one split), so the product lands in place
    P->has_fwg = gr != nullptr;
    if (gr && (!desc_fc_wgrad(&P->fwg[f], h->fc[f], dz[f], fin[f], gr, B, ns, h->status) ||
               P->fwg[f].args.splits != 1))
      P->has_fwg = false;
  }
  if (h->scratch) {
    const GemmDesc* all[] = {&P->ff[0], &P->ff[1], &P->ff[2], &P->fd[0], &P->fd[1],
                             &P->fd[2], &P->fw[0], &P->fw[1], &P->fw[2]};
    for (const GemmDesc* d : all)
      if (desc_f32_need(*d) > h->scratch_floats) return set_err(h, "scratch too small for plan");
    for (int l = 0; l < 5; ++l)
      if (P->cw[l].f32_need() > h->scratch_floats)
        return set_err(h, "scratch too small for plan");
  }
  P->ok = true;
  return true;
}

// Carve every buffer of the handle out of the workspace (or size it).
size_t carve(alexnet* h, void* base) {
  if (base) h->guards.clear();
  Carver c(base, base ? &h->guards : nullptr);
  const alexnet_config& cfg = h->cfg;
  const int B = cfg.batch_max;
  const size_t n = h->n_params;
  float* pv = c.take<float>(2 * n);
  h->params = pv;
  h->vel = pv ? pv + n : nullptr;
  h->grads = cfg.keep_grads ? c.take<float>(n) : nullptr;
  h->hp = c.take<HParams>(1);
  h->status = c.take<int>(4);
  h->loss_dev = c.take<float>(4);
  h->loss_rows = c.take<float>(B > 16 ? B : 16);
  h->labels_buf = c.take<int32_t>(B > 16 ? B : 16);
  h->logits = c.take<float>(static_cast<size_t>(B) * kClasses);
  h->probs = c.take<float>(static_cast<size_t>(B) * kClasses);
  if (cfg.dtype == ALEXNET_FP32) {
    size_t mx = 0;
    for (int l = 0; l < 5; ++l) {
      const ConvL& L = h->conv[l];
      const size_t e = static_cast<size_t>(B) * L.Ho * L.Ho * L.Cout;
      if (e > mx) mx = e;
    }
    const size_t xin = static_cast<size_t>(B) * 227 * 227 * 3;
    if (xin > mx) mx = xin;
    h->f_act = mx;
    h->fa = c.take<float>(mx);
    h->fb = c.take<float>(mx);
    size_t wmax = 0;
    for (int l = 0; l < 5; ++l) wmax = h->w_len[l] > wmax ? h->w_len[l] : wmax;
    h->fwt = c.take<float>(wmax);
    return c.off;
  }
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    h->wf[l] = c.take<bf16>(static_cast<size_t>(L.Cout) * L.Kdim());
    if (l > 0) h->wd[l] = c.take<bf16>(h->w_len[l]);
  }
  for (int f = 0; f < 3; ++f) h->wf[5 + f] = c.take<bf16>(h->w_len[5 + f]);
  h->xin = c.take<bf16>(static_cast<size_t>(B) * 227 * 227 * 3);
  h->xs = c.take<bf16>(static_cast<size_t>(B) * 57 * 57 * 64);
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    const size_t e = static_cast<size_t>(B) * L.Ho * L.Ho * L.Cout;
    const size_t ep = static_cast<size_t>(B) * L.P * L.P * L.Cout;
    h->a[l] = c.take<bf16>(e);
    h->da[l] = c.take<bf16>(e);
    if (L.lrn) {
      h->lo[l] = c.take<bf16>(e);
      h->dl[l] = c.take<bf16>(e);
    }
    if (L.pool) {
      h->p[l] = c.take<bf16>(ep);
      h->am[l] = c.take<uint8_t>(ep);
      h->dp[l] = c.take<bf16>(ep);
    }
  }
  h->dp5 = h->dp[4];
  h->f6 = c.take<bf16>(static_cast<size_t>(B) * 4096);
  h->f7 = c.take<bf16>(static_cast<size_t>(B) * 4096);
  h->dlogits = c.take<bf16>(static_cast<size_t>(B) * kClasses);
  h->d7 = c.take<bf16>(static_cast<size_t>(B) * 4096);
  h->d6 = c.take<bf16>(static_cast<size_t>(B) * 4096);
  // column-sum partials for the conv bias gradients, one region per layer
  // (all five updates run in one launch at the end of the backward pass):
  // the most rows any producer writes (column sums of da, the fused pool +
  // normalisation backward, the pool backward) x cols
  size_t cp = 0;
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    size_t rows = static_cast<size_t>(colsum_chunks(1LL * B * L.Ho * L.Ho));
    rows = std::max(rows, static_cast<size_t>(
                              pool_lrn_bwd_parts(B, L.Ho, L.Ho, L.Cout, cfg.pool_size)));
    rows = std::max(rows, static_cast<size_t>(pool_bwd_parts(B, L.Ho, L.Ho, L.Cout)));
    h->cpart_off[l] = cp;
    cp += (rows * L.Cout + 63) / 64 * 64;
  }
  h->cpart_floats = cp;
  h->cpart = c.take<float>(cp);
  // fp32 scratch: split-K partials and FC weight gradients, sized by the
  // plans at batch_max (smaller batches never need more)
  {
    alexnet tmp;
    tmp.cfg = h->cfg;
    tmp.num_sms = h->num_sms;
    build_geometry(&tmp);
    Plan P;
    g_dry_tmaps = true;
    const bool ok = build_plan(&tmp, B, &P);
    g_dry_tmaps = false;
    size_t need = 1;
    if (ok) {
      const GemmDesc* all[] = {&P.ff[0], &P.ff[1], &P.ff[2], &P.fd[0], &P.fd[1],
                               &P.fd[2], &P.fw[0], &P.fw[1], &P.fw[2]};
      for (const GemmDesc* d : all) need = desc_f32_need(*d) > need ? desc_f32_need(*d) : need;
      for (int l = 0; l < 5; ++l) need = P.cw[l].f32_need() > need ? P.cw[l].f32_need() : need;
    }
    h->scratch_floats = need;
    h->scratch = c.take<float>(need);
  }
  return c.off;
}

void write_hp(alexnet* h, float lr, cudaStream_t s) {
  h->hp_host.lr = lr;
  h->hp_host.momentum = h->cfg.momentum;
  h->hp_host.weight_decay = h->cfg.weight_decay;
  h->hp_host.dropout_p = h->cfg.dropout_p;
  h->hp_host.step = static_cast<uint32_t>(h->step);
  h->hp_host.seed_lo = static_cast<uint32_t>(h->cfg.seed);
  h->hp_host.seed_hi = static_cast<uint32_t>(h->cfg.seed >> 32);
  const double t = static_cast<double>(h->cfg.dropout_p) * 4294967296.0 + 0.5;
  h->hp_host.drop_thresh = t >= 4294967295.0 ? 0xFFFFFFFFu : static_cast<uint32_t>(t);
  h->hp_host.update = h->grads_only ? 0u : 1u;
  h->hp_host.row_offset = h->grads_only ? h->row_offset : 0u;
  launch_write_hparams(h->hp, h->hp_host, s);
}

ConvMap conv_map(const alexnet* h, int l) {
  const ConvL& L = h->conv[l];
  ConvMap m;
  m.Cout = L.Cout;
  m.K = L.K;
  m.Cg = L.Cin / L.groups;
  m.groups = L.groups;
  m.s2d = l == 0 ? 1 : 0;
  m.P = L.Pch();
  return m;
}

void refresh_shadows(alexnet* h, cudaStream_t s) {
  if (h->cfg.dtype != ALEXNET_BF16) return;
  for (int l = 0; l < 5; ++l)
    launch_conv_shadows(h->params + h->w_off[l], conv_map(h, l), h->wf[l], h->wd[l], s);
  for (int f = 5; f < 8; ++f) launch_f32_to_bf16(h->params + h->w_off[f], h->wf[f], h->w_len[f], s);
}

Plan* get_plan(alexnet* h, int B) {
  auto it = h->plans.find(B);
  if (it != h->plans.end()) return &it->second;
  Plan P;
  if (!build_plan(h, B, &P)) return nullptr;
  auto r = h->plans.emplace(B, P);
  return &r.first->second;
}

#define ALX_TRY(expr, where)                                                 \
  do {                                                                       \
    cudaError_t e_ = (expr);                                                 \
    if (e_ != cudaSuccess) return cuda_status(h, e_, where);                 \
  } while (0)

cudaError_t launch_any(const GemmDesc& d, cudaStream_t s) { return gemm_launch(d, s); }
cudaError_t launch_any(const ConvPlan& d, cudaStream_t s) { return conv_plan_launch(d, s); }

template <typename D>
cudaError_t run_gemm(alexnet* h, const D& d, double flops, cudaStream_t s, int kind = 0) {
  if (!h->stats_on || !h->rec) return launch_any(d, s);
  alexnet::StepRec& R = *h->rec;
  while (R.used + 2 > R.ev.size()) {
    cudaEvent_t e;
    cudaError_t r = cudaEventCreate(&e);
    if (r != cudaSuccess) return r;
    R.ev.push_back(e);
  }
  cudaEvent_t e0 = R.ev[R.used], e1 = R.ev[R.used + 1];
  R.used += 2;
  // inside a capture the records become event nodes of the graph
  const unsigned flags = h->capturing ? cudaEventRecordExternal : cudaEventRecordDefault;
  cudaEventRecordWithFlags(e0, s, flags);
  cudaError_t r = launch_any(d, s);
  cudaEventRecordWithFlags(e1, s, flags);
  R.gemm_launches += 1;
  R.gemm_flops += flops;
  R.flops.push_back(flops);
  R.kind.push_back(kind);
  return r;
}

// x == nullptr: the space-to-depth input xs is already in place.
alexnet_status forward_bf16(alexnet* h, const bf16* x, int B, int dropout_mode, float* logits,
                            cudaStream_t s, Plan* P) {
  if (x) launch_s2d(x, h->xs, B, s);
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    ALX_TRY(run_gemm(h, P->cf[l], P->conv_flops[l], s), "conv forward launch");
    if (L.lrn && L.pool &&
        launch_lrn_pool_fwd(h->a[l], h->keep ? h->lo[l] : nullptr, h->p[l], h->am[l], B, L.Ho,
                            L.Ho, L.Cout, h->cfg.pool_size, h->cfg.lrn_k, h->cfg.lrn_alpha,
                            h->cfg.lrn_beta, s))
      continue;
    const bf16* cur = h->a[l];
    if (L.lrn) {
      launch_lrn_fwd(h->a[l], h->lo[l], 1LL * B * L.Ho * L.Ho, L.Cout, h->cfg.lrn_n, h->cfg.lrn_k,
                     h->cfg.lrn_alpha, h->cfg.lrn_beta, s);
      cur = h->lo[l];
    }
    if (L.pool)
      launch_pool_fwd(cur, h->p[l], h->am[l], B, L.Ho, L.Ho, L.Cout, h->cfg.pool_size, 2, s);
  }
  bf16* fout[2] = {h->f6, h->f7};
  for (int f = 0; f < 3; ++f) {
    ALX_TRY(run_gemm(h, P->ff[f], P->fc_flops[f], s, 1), "fc forward launch");
    const float* bias = h->params + h->b_off[5 + f];
    if (f < 2)
      launch_fc_finalize(h->scratch, P->ff[f].args.splits, B, h->fc[f].Out, bias, 1, dropout_mode,
                         6 + f, h->hp, fout[f], nullptr, s);
    else
      launch_fc_finalize(h->scratch, P->ff[f].args.splits, B, h->fc[f].Out, bias, 0, 0, 8, h->hp,
                         nullptr, logits, s);
  }
  return cuda_status(h, cudaGetLastError(), "forward");
}

alexnet_status forward_f32(alexnet* h, const float* x, int B, float* logits, cudaStream_t s) {
  const float* cur = x;
  float* bufs[2] = {h->fa, h->fb};
  int which = 0;
  for (int l = 0; l < 5; ++l) {
    const ConvL& L = h->conv[l];
    launch_conv_wt_f32(h->params + h->w_off[l], h->fwt, L.Cout, L.K, L.Cin / L.groups, L.groups, s);
    float* y = bufs[which];
    launch_conv_fwd_f32(cur, h->fwt, h->params + h->b_off[l], y, B, L.H, L.H, L.Cin, L.Cout, L.K,
                        L.stride, L.pad, L.groups, L.Ho, L.Ho, s);
    which ^= 1;
    cur = y;
    if (L.lrn) {
      float* z = bufs[which];
      launch_lrn_fwd_f32(cur, z, 1LL * B * L.Ho * L.Ho, L.Cout, 5, h->cfg.lrn_k, h->cfg.lrn_alpha,
                         h->cfg.lrn_beta, s);
      which ^= 1;
      cur = z;
    }
    if (L.pool) {
      float* z = bufs[which];
      launch_pool_fwd_f32(cur, z, B, L.Ho, L.Ho, L.Cout, h->cfg.pool_size, 2, s);
      which ^= 1;
      cur = z;
    }
  }
  const float scale = h->cfg.dropout_on ? 1.f - h->cfg.dropout_p : 1.f;
  for (int f = 0; f < 3; ++f) {
    float* y = f < 2 ? bufs[which] : logits;
    launch_fc_fwd_f32(cur, h->params + h->w_off[5 + f], h->params + h->b_off[5 + f], y, B,
                      h->fc[f].In, h->fc[f].Out, f < 2 ? 1 : 0, f < 2 ? scale : 1.f, s);
    if (f < 2) {
      which ^= 1;
      cur = y;
    }
  }
  return cuda_status(h, cudaGetLastError(), "forward fp32");
}

// Forward, loss and the FC layers' backward (with their update, unless the
// handle runs a gradient-only step).
// The second stream for the weight gradients and updates (created with its
// events on first use); nullptr when the overlap is off, or while per-GEMM
// timing is on (each GEMM is then timed alone).
cudaError_t side_stream(alexnet* h, cudaStream_t* out) {
  *out = nullptr;
  if (!h->overlap_wgrad || h->stats_on) return cudaSuccess;
  if (!h->side) {
    cudaError_t e = cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking);
    auto ev = [&](cudaEvent_t* x) {
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(x, cudaEventDisableTiming);
    };
    for (int l = 0; l < 5; ++l) {
      ev(&h->ev_dy[l]);
      ev(&h->ev_dg[l]);
    }
    for (int f = 0; f < 3; ++f) {
      ev(&h->ev_fdz[f]);
      ev(&h->ev_fdg[f]);
    }
    ev(&h->ev_join);
    ev(&h->ev_fjoin);
    if (e != cudaSuccess) return e;
  }
  *out = h->side;
  return cudaSuccess;
}

alexnet_status train_fc_part(alexnet* h, const bf16* x, const int32_t* labels, int B, float* loss,
                             cudaStream_t s, Plan* P) {
  const alexnet_config& cfg = h->cfg;
  alexnet_status st = forward_bf16(h, x, B, cfg.dropout_on ? 1 : 0, h->logits, s, P);
  // (x == nullptr: the caller converted the input already)
  if (st != ALEXNET_OK) return st;
  launch_softmax_ce(h->logits, labels, B, kClasses, nullptr, h->dlogits, h->loss_rows, h->status,
                    s);
  launch_loss_mean(h->loss_rows, B, h->loss_dev, loss, s);
  float* gr = h->grads;
  auto gptr = [&](size_t off) { return gr ? gr + off : nullptr; };
  // FC8, FC7, FC6: data gradient (old weights), then weight gradient + SGD.
  // With the update in the weight-gradient epilogue (or gradients only) the
  // weight gradient, update and bias update go to the second stream once dz
  // is complete, the update after the data gradient that reads the layer's
  // old weights (the separate-kernel update shares the split-K scratch with
  // the data gradients and stays on one stream).
  const bf16* dz[3] = {h->d6, h->d7, h->dlogits};
  bf16* dxo[3] = {h->dp5, h->d6, h->d7};
  const bf16* mask[3] = {nullptr, h->f6, h->f7};
  cudaStream_t side = nullptr;
  if (h->fc_fused || h->grads_only) ALX_TRY(side_stream(h, &side), "side stream");
  for (int f = 2; f >= 0; --f) {
    const FcL& F = h->fc[f];
    cudaStream_t ws = s;
    if (side) {
      ALX_TRY(cudaEventRecord(h->ev_fdz[f], s), "fork");
      ALX_TRY(cudaStreamWaitEvent(side, h->ev_fdz[f], 0), "fork");
      ws = side;
    }
    ALX_TRY(run_gemm(h, P->fd[f], P->fc_flops[f], s, 1), "fc dgrad launch");
    if (side) ALX_TRY(cudaEventRecord(h->ev_fdg[f], s), "data gradient done");
    launch_dgrad_finalize(h->scratch, P->fd[f].args.splits, B, F.In, mask[f], dxo[f], s);
    if (h->grads_only) {
      ALX_TRY(run_gemm(h, P->fwg[f], P->fc_flops[f], ws, 2), "fc wgrad launch");
    } else if (h->fc_fused) {
      // HBM-bound (the update moves 18 bytes per weight against 256 MMA
      // FLOPs): launched outside the per-GEMM tensor-roofline records
      if (side) ALX_TRY(cudaStreamWaitEvent(side, h->ev_fdg[f], 0), "update after dgrad");
      ALX_TRY(launch_any(P->fws[f], ws), "fc wgrad + update launch");
    } else {
      ALX_TRY(run_gemm(h, P->fw[f], P->fc_flops[f], s, 2), "fc wgrad launch");
      launch_sgd_dense(h->params + h->w_off[5 + f], h->vel + h->w_off[5 + f], h->scratch,
                       h->w_len[5 + f], h->wf[5 + f], gptr(h->w_off[5 + f]), h->hp, s);
    }
    launch_sgd_bias_rows(h->params + h->b_off[5 + f], h->vel + h->b_off[5 + f], dz[f], B, F.Out,
                         gptr(h->b_off[5 + f]), h->hp, ws);
  }
  // gradients only: the FC gradients are complete when this part ends (the
  // caller's event marks them); in a training step the side stream carries
  // on into the convolutions' part and is joined at its end
  if (side && h->grads_only) {
    ALX_TRY(cudaEventRecord(h->ev_fjoin, side), "join");
    ALX_TRY(cudaStreamWaitEvent(s, h->ev_fjoin, 0), "join");
  }
  return cuda_status(h, cudaGetLastError(), "train step (FC part)");
}

// The convolutions' backward and update (or gradients only), top down.
alexnet_status train_conv_part(alexnet* h, int B, cudaStream_t s, Plan* P) {
  const alexnet_config& cfg = h->cfg;
  float* gr = h->grads;
  auto gptr = [&](size_t off) { return gr ? gr + off : nullptr; };
  // Per conv layer, top down: bias update (its column sums come from the
  // pool (+ normalisation) backward that produced da where it made them,
  // else from da), data gradient into the layer below (and that layer's
  // pool/LRN/ReLU backward), weight gradient and update.
  bool fused_bwd[5] = {false, false, false, false, false};
  int bias_parts[5] = {0, 0, 0, 0, 0};
  cudaStream_t side = nullptr;
  ALX_TRY(side_stream(h, &side), "side stream");
  // pool5 backward straight into conv5's pre-activation gradient, with
  // conv5's bias column sums
  {
    const ConvL& L = h->conv[4];
    float* part = h->cpart + h->cpart_off[4];
    int parts = launch_pool_relu_bwd_staged(h->dp5, h->am[4], h->a[4], h->da[4], B, L.Ho, L.Ho,
                                            L.Cout, cfg.pool_size, part, h->status, s);
    if (parts == 0)
      parts = launch_pool_bwd(h->dp5, h->am[4], h->p[4], h->da[4], B, L.Ho, L.Ho, L.Cout,
                              cfg.pool_size, 2, 1, s, part);
    if (parts > 0) {
      fused_bwd[4] = true;
      bias_parts[4] = parts;
    }
  }
  for (int l = 4; l >= 0; --l) {
    const ConvL& L = h->conv[l];
    const long long rows = 1LL * B * L.Ho * L.Ho;
    // dY of layer l is complete: its weight gradient (and, where no pool
    // backward made them, its bias column sums) may start beside
    cudaStream_t ws = s;
    if (side) {
      ALX_TRY(cudaEventRecord(h->ev_dy[l], s), "fork");
      ALX_TRY(cudaStreamWaitEvent(side, h->ev_dy[l], 0), "fork");
      ws = side;
    }
    if (!fused_bwd[l]) {
      launch_colsum_partial(h->da[l], rows, L.Cout, h->cpart + h->cpart_off[l], ws);
      bias_parts[l] = colsum_chunks(rows);
    }
    if (l > 0) {
      ALX_TRY(run_gemm(h, P->cd[l], P->conv_flops[l], s), "conv dgrad launch");
      if (side) ALX_TRY(cudaEventRecord(h->ev_dg[l], s), "data gradient done");
      const ConvL& Q = h->conv[l - 1];
      if (Q.pool) {
        // dp[l-1] = d(pooled map) -> through the pool (and LRN) to da[l-1]
        if (Q.lrn) {
          // pool + normalisation + ReLU backward in one pass when the shape
          // allows it (with layer l-1's bias column sums), else pool
          // backward now and normalisation below
          const int rows = launch_pool_lrn_bwd(
              h->dp[l - 1], h->am[l - 1], h->a[l - 1], h->keep ? h->dl[l - 1] : nullptr,
              h->da[l - 1], B, Q.Ho, Q.Ho, Q.Cout, cfg.pool_size, cfg.lrn_k, cfg.lrn_alpha,
              cfg.lrn_beta, h->cpart + h->cpart_off[l - 1], h->status, s);
          fused_bwd[l - 1] = rows > 0;
          if (rows > 0)
            bias_parts[l - 1] = rows;
          else
            launch_pool_bwd(h->dp[l - 1], h->am[l - 1], h->p[l - 1], h->dl[l - 1], B, Q.Ho, Q.Ho,
                            Q.Cout, cfg.pool_size, 2, 0, s);
        } else {
          // pool + ReLU backward (the no-normalisation variant), with layer
          // l-1's bias column sums where the staged kernel takes the shape
          float* part = h->cpart + h->cpart_off[l - 1];
          int rows = launch_pool_relu_bwd_staged(h->dp[l - 1], h->am[l - 1], h->a[l - 1],
                                                 h->da[l - 1], B, Q.Ho, Q.Ho, Q.Cout,
                                                 cfg.pool_size, part, h->status, s);
          if (rows == 0)
            rows = launch_pool_bwd(h->dp[l - 1], h->am[l - 1], h->p[l - 1], h->da[l - 1], B,
                                   Q.Ho, Q.Ho, Q.Cout, cfg.pool_size, 2, 1, s, part);
          fused_bwd[l - 1] = rows > 0;
          if (rows > 0) bias_parts[l - 1] = rows;
        }
      }
    }
    if (l > 0) {
      const ConvL& Q = h->conv[l - 1];
      if (Q.pool && Q.lrn && !fused_bwd[l - 1])
        launch_lrn_bwd(h->a[l - 1], h->dl[l - 1], h->da[l - 1], 1LL * B * Q.Ho * Q.Ho, Q.Cout,
                       cfg.lrn_n, cfg.lrn_k, cfg.lrn_alpha, cfg.lrn_beta, s);
    }
    // weight gradient (split partials in scratch, one layer at a time on
    // the side stream) and update; the update rewrites the bf16 weights the
    // data gradient above reads, so it waits for it
    ALX_TRY(run_gemm(h, P->cw[l], P->conv_flops[l], ws), "conv wgrad launch");
    if (side && l > 0) ALX_TRY(cudaStreamWaitEvent(side, h->ev_dg[l], 0), "update after dgrad");
    launch_sgd_conv(h->params + h->w_off[l], h->vel + h->w_off[l], h->scratch,
                    P->cw[l].splits(), conv_map(h, l), h->wf[l], h->need_wd ? h->wd[l] : nullptr,
                    gptr(h->w_off[l]), h->hp, ws);
  }
  if (side) {
    ALX_TRY(cudaEventRecord(h->ev_join, side), "join");
    ALX_TRY(cudaStreamWaitEvent(s, h->ev_join, 0), "join");
  }
  // the five conv bias updates, from their column-sum partials
  BiasJobs jobs{};
  jobs.count = 5;
  for (int l = 0; l < 5; ++l) {
    BiasJob& J = jobs.j[l];
    J.b = h->params + h->b_off[l];
    J.v = h->vel + h->b_off[l];
    J.partial = h->cpart + h->cpart_off[l];
    J.chunks = bias_parts[l];
    J.n = h->conv[l].Cout;
    J.grads_out = gptr(h->b_off[l]);
  }
  launch_sgd_bias_jobs(jobs, h->hp, s);
  return cuda_status(h, cudaGetLastError(), "train step");
}

alexnet_status train_bf16(alexnet* h, const bf16* x, const int32_t* labels, int B, float* loss,
                          cudaStream_t s, Plan* P) {
  alexnet_status st = train_fc_part(h, x, labels, B, loss, s, P);
  if (st != ALEXNET_OK) return st;
  return train_conv_part(h, B, s, P);
}

// Runs body(stream) for graph `key`: captured into a CUDA graph the first
// time, replayed afterwards (direct launches when graphs are off).
template <typename F>
alexnet_status replay(alexnet* h, int key, cudaStream_t s, F&& body) {
  if (!h->use_graphs) {
    h->direct_rec.reset();
    h->rec = h->stats_on ? &h->direct_rec : nullptr;
    const alexnet_status st = body(s);
    h->rec = nullptr;
    if (h->stats_on) h->last_rec = &h->direct_rec;
    return st;
  }
  auto it = h->train_graphs.find(key);
  if (it == h->train_graphs.end()) {
    if (!h->cap_stream)
      ALX_TRY(cudaStreamCreateWithFlags(&h->cap_stream, cudaStreamNonBlocking), "capture stream");
    ALX_TRY(cudaStreamBeginCapture(h->cap_stream, cudaStreamCaptureModeThreadLocal),
            "begin capture");
    const int64_t c0 = launch_counter();
    h->rec = h->stats_on ? &h->graph_rec[key] : nullptr;
    h->capturing = true;
    const alexnet_status st = body(h->cap_stream);
    h->capturing = false;
    h->rec = nullptr;
    // captured kernels are counted when a replay runs them, not now
    h->graph_kernels[key] = launch_counter() - c0;
    count_launch_n(-(launch_counter() - c0));
    cudaGraph_t g = nullptr;
    const cudaError_t ce = cudaStreamEndCapture(h->cap_stream, &g);
    if (st != ALEXNET_OK) {
      if (g) cudaGraphDestroy(g);
      return st;
    }
    ALX_TRY(ce, "end capture");
    cudaGraphExec_t ex = nullptr;
    const cudaError_t ie = cudaGraphInstantiate(&ex, g, 0);
    cudaGraphDestroy(g);
    ALX_TRY(ie, "graph instantiate");
    it = h->train_graphs.emplace(key, ex).first;
  }
  ALX_TRY(cudaGraphLaunch(it->second, s), "graph launch");
  count_launch_n(h->graph_kernels[key]);
  if (h->stats_on) h->last_rec = &h->graph_rec[key];
  return ALEXNET_OK;
}

}  // namespace

// ======================================================================
// C ABI
// ======================================================================
extern "C" {

void alexnet_default_config(alexnet_config* c) {
  if (!c) return;
  memset(c, 0, sizeof(*c));
  c->batch_max = 128;
  c->dtype = ALEXNET_BF16;
  c->grouped = 1;
  c->seed = 0x5EEDULL;
  c->momentum = 0.9f;
  c->weight_decay = 5e-4f;
  c->dropout_p = 0.5f;
  c->lrn_k = 2.f;
  c->lrn_alpha = 1e-4f;
  c->lrn_beta = 0.75f;
  c->lrn_n = 5;
  c->lrn_on = 1;
  c->pool_size = 3;
  c->dropout_on = 1;
  c->keep_grads = 0;
}

int64_t alexnet_param_count(const alexnet_config* cfg) {
  if (!valid_config(cfg)) return -1;
  alexnet tmp;
  tmp.cfg = *cfg;
  build_geometry(&tmp);
  return static_cast<int64_t>(tmp.n_params);
}

size_t alexnet_workspace_bytes(const alexnet_config* cfg) {
  if (!valid_config(cfg)) return 0;
  alexnet tmp;
  tmp.cfg = *cfg;
  build_geometry(&tmp);
  return carve(&tmp, nullptr) + 256;
}

alexnet_status alexnet_create(const alexnet_config* cfg, void* workspace, size_t bytes,
                              void* stream, alexnet_t** out) {
  if (!out) return ALEXNET_ERR_INVALID_ARG;
  *out = nullptr;
  if (!valid_config(cfg)) {
    g_create_error = "invalid config";
    return ALEXNET_ERR_INVALID_ARG;
  }
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255)) {
    g_create_error = "workspace must be a 256-byte aligned device pointer";
    return ALEXNET_ERR_INVALID_ARG;
  }
  const size_t need = alexnet_workspace_bytes(cfg);
  if (bytes < need) {
    g_create_error = "workspace too small";
    return ALEXNET_ERR_INVALID_ARG;
  }
  alexnet* h = new alexnet();
  h->cfg = *cfg;
  h->ws = static_cast<char*>(workspace);
  h->ws_bytes = bytes;
  int dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, dev);
  build_geometry(h);
  carve(h, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  cudaError_t pe = box_prepare();
  if (pe == cudaSuccess) pe = gemm_prepare();
  if (pe != cudaSuccess) {
    g_create_error = std::string("create: ") + cudaGetErrorString(pe);
    delete h;
    return ALEXNET_ERR_CUDA;
  }
  // initial parameters ([S] 3.4 "Training Procedure Details")
  const int bias_one[8] = {0, 1, 0, 1, 1, 1, 1, 0};
  for (int l = 0; l < 8; ++l) {
    launch_init_normal(h->params + h->w_off[l], h->w_len[l], 0.01f, cfg->seed,
                       static_cast<uint32_t>(l), s);
    launch_fill(h->params + h->b_off[l], h->b_len[l], bias_one[l] ? 1.f : 0.f, s);
  }
  launch_fill(h->vel, h->n_params, 0.f, s);
  cudaError_t e = cudaMemsetAsync(h->status, 0, sizeof(int), s);
  for (size_t i = 0; i < h->guards.size() && e == cudaSuccess; ++i)
    e = cudaMemsetAsync(h->ws + h->guards[i], kCanaryByte, kCanaryBytes, s);
  for (int l = 0; l < 5 && e == cudaSuccess && h->cfg.dtype == ALEXNET_BF16; ++l)
    e = cudaMemsetAsync(h->wf[l], 0, sizeof(bf16) * h->conv[l].Cout * h->conv[l].Kdim(), s);
  refresh_shadows(h, s);
  write_hp(h, 0.f, s);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) {
    g_create_error = std::string("create: ") + cudaGetErrorString(e);
    delete h;
    return ALEXNET_ERR_CUDA;
  }
  *out = h;
  return ALEXNET_OK;
}

alexnet_status alexnet_forward(alexnet_t* h, const void* x, int B, alexnet_mode mode,
                               float* logits, float* probs, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!x || !logits || B < 1 || B > h->cfg.batch_max ||
      (mode != ALEXNET_TRAIN && mode != ALEXNET_INFERENCE) ||
      (reinterpret_cast<uintptr_t>(x) & 15)) {
    h->err = "forward: invalid argument (x must be a 16-byte aligned device pointer)";
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  alexnet_status st;
  if (h->cfg.dtype == ALEXNET_FP32) {
    if (mode == ALEXNET_TRAIN && h->cfg.dropout_on) {
      h->err = "forward: the fp32 path serves inference only";
      return ALEXNET_ERR_UNSUPPORTED;
    }
    st = forward_f32(h, static_cast<const float*>(x), B, logits, s);
  } else {
    Plan* P = get_plan(h, B);
    if (!P) return ALEXNET_ERR_CUDA;
    const int64_t l0 = launch_counter();
    write_hp(h, 0.f, s);
    const int dm = !h->cfg.dropout_on ? 0 : (mode == ALEXNET_TRAIN ? 1 : 2);
    h->direct_rec.reset();
    h->rec = h->stats_on ? &h->direct_rec : nullptr;
    st = forward_bf16(h, static_cast<const bf16*>(x), B, dm, logits, s, P);
    h->rec = nullptr;
    if (h->stats_on) {
      h->last_rec = &h->direct_rec;
      h->last_launches = launch_counter() - l0;
      h->stats_stream = s;
    }
  }
  if (st != ALEXNET_OK) return st;
  if (probs)
    launch_softmax_ce(logits, nullptr, B, kClasses, probs, nullptr, nullptr, h->status, s);
  if (logits != h->logits)
    cudaMemcpyAsync(h->logits, logits, sizeof(float) * B * kClasses, cudaMemcpyDeviceToDevice, s);
  return cuda_status(h, cudaGetLastError(), "forward");
}

alexnet_status alexnet_train_step(alexnet_t* h, const void* x, const int32_t* labels, int B,
                                  float lr, float* loss, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!x || !labels || B < 1 || B > h->cfg.batch_max || !(lr >= 0.f) ||
      (reinterpret_cast<uintptr_t>(x) & 15)) {
    h->err = "train_step: invalid argument (x must be a 16-byte aligned device pointer)";
    return ALEXNET_ERR_INVALID_ARG;
  }
  if (h->cfg.dtype != ALEXNET_BF16) {
    h->err = "train_step: training runs on the bf16 path only";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  Plan* P = get_plan(h, B);
  if (!P) return ALEXNET_ERR_CUDA;
  // Everything that depends on the call's arguments runs outside the graph:
  // the hyper-parameters (lr, step), the input conversion, the labels copy
  // and the loss copy.  The graph itself only touches the workspace.
  write_hp(h, lr, s);
  launch_s2d(static_cast<const bf16*>(x), h->xs, B, s);
  ALX_TRY(cudaMemcpyAsync(h->labels_buf, labels, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, s),
          "train_step labels");
  const int64_t l0 = launch_counter();
  const int key = 64 * B + (h->overlap_wgrad ? 32 : 0) + (h->fc_fused ? 4 : 0) +
                  (h->keep ? 2 : 0) + (h->stats_on ? 1 : 0);
  const alexnet_status st = replay(h, key, s, [&](cudaStream_t cs) {
    return train_bf16(h, nullptr, h->labels_buf, B, nullptr, cs, P);
  });
  if (h->stats_on) {
    h->last_launches = launch_counter() - l0;
    h->stats_stream = s;
  }
  if (st != ALEXNET_OK) return st;
  if (loss)
    ALX_TRY(cudaMemcpyAsync(loss, h->loss_dev, sizeof(float), cudaMemcpyDeviceToDevice, s),
            "train_step loss");
  h->step += 1;
  return cuda_status(h, cudaGetLastError(), "train step");
}

alexnet_status alexnet_train_grads(alexnet_t* h, const void* x, const int32_t* labels, int B,
                                   int64_t image_offset, float* loss, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!x || !labels || B < 1 || B > h->cfg.batch_max || image_offset < 0 ||
      image_offset > 0x7FFFFFFF - B || (reinterpret_cast<uintptr_t>(x) & 15)) {
    h->err = "train_grads: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  if (h->cfg.dtype != ALEXNET_BF16 || !h->grads) {
    h->err = "train_grads: needs a bf16 handle created with keep_grads";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  Plan* P = get_plan(h, B);
  if (!P) return ALEXNET_ERR_CUDA;
  if (!P->has_fwg) {
    h->err = "train_grads: the FC weight gradients do not fit one K-slice at this batch";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  if (!h->fc_event)
    ALX_TRY(cudaEventCreateWithFlags(&h->fc_event, cudaEventDisableTiming), "fc event");
  h->grads_only = true;
  h->row_offset = static_cast<uint32_t>(image_offset);
  write_hp(h, 0.f, s);
  launch_s2d(static_cast<const bf16*>(x), h->xs, B, s);
  alexnet_status st = ALEXNET_OK;
  cudaError_t e = cudaMemcpyAsync(h->labels_buf, labels, sizeof(int32_t) * B,
                                  cudaMemcpyDeviceToDevice, s);
  const bool stats = h->stats_on;
  h->stats_on = false;
  // two graphs: forward + FC backward, then the convolutions' backward, with
  // the FC-gradients event recorded between them
  const int base = 64 * B + (h->overlap_wgrad ? 32 : 0) + (h->keep ? 2 : 0) + 16;
  if (e == cudaSuccess)
    st = replay(h, base, s, [&](cudaStream_t cs) {
      return train_fc_part(h, nullptr, h->labels_buf, B, nullptr, cs, P);
    });
  if (e == cudaSuccess && st == ALEXNET_OK) e = cudaEventRecord(h->fc_event, s);
  if (e == cudaSuccess && st == ALEXNET_OK)
    st = replay(h, base + 8, s, [&](cudaStream_t cs) { return train_conv_part(h, B, cs, P); });
  h->stats_on = stats;
  h->grads_only = false;
  h->row_offset = 0;
  if (e != cudaSuccess) return cuda_status(h, e, "train_grads");
  if (st != ALEXNET_OK) return st;
  if (loss)
    ALX_TRY(cudaMemcpyAsync(loss, h->loss_dev, sizeof(float), cudaMemcpyDeviceToDevice, s),
            "train_grads loss");
  return cuda_status(h, cudaGetLastError(), "train_grads");
}

alexnet_status alexnet_stream_wait_fc_grads(alexnet_t* h, void* stream) {
  if (!h || !h->fc_event) return ALEXNET_ERR_INVALID_ARG;
  return cuda_status(h, cudaStreamWaitEvent(static_cast<cudaStream_t>(stream), h->fc_event, 0),
                     "stream_wait_fc_grads");
}

alexnet_status alexnet_sgd_range(alexnet_t* h, int64_t offset, int64_t count, const float* g,
                                 float grad_scale, float lr, void* stream) {
  if (!h || !g || offset < 0 || count < 0 ||
      offset + count > static_cast<int64_t>(h->n_params) || !(lr >= 0.f) ||
      h->cfg.dtype != ALEXNET_BF16)
    return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  if (count == 0) return ALEXNET_OK;
  launch_sgd_range(h->params + offset, h->vel + offset, g, count, grad_scale, lr,
                   h->cfg.momentum, h->cfg.weight_decay, s);
  return cuda_status(h, cudaGetLastError(), "sgd_range");
}

alexnet_status alexnet_params_updated(alexnet_t* h, void* stream) {
  if (!h || h->cfg.dtype != ALEXNET_BF16) return ALEXNET_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  refresh_shadows(h, s);
  h->step += 1;
  return cuda_status(h, cudaGetLastError(), "params_updated");
}

alexnet_status alexnet_device_buffer(alexnet_t* h, int which, void** ptr, int64_t* count) {
  if (!h || !ptr || !count) return ALEXNET_ERR_INVALID_ARG;
  *ptr = nullptr;
  *count = 0;
  float* p = which == 0 ? h->params : (which == 1 ? h->vel : (which == 2 ? h->grads : nullptr));
  if (!p) return ALEXNET_ERR_INVALID_ARG;
  *ptr = p;
  *count = static_cast<int64_t>(h->n_params);
  return ALEXNET_OK;
}

alexnet_status alexnet_augment(alexnet_t* h, const uint8_t* src, int B, const float* mean,
                               const float* pca_vec, const float* pca_val, void* x_out,
                               void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!src || !mean || !pca_vec || !pca_val || !x_out || B < 1) {
    h->err = "augment: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  write_hp(h, h->hp_host.lr, s);
  launch_augment(src, B, mean, pca_vec, pca_val, h->hp, static_cast<bf16*>(x_out), s);
  return cuda_status(h, cudaGetLastError(), "augment");
}

alexnet_status alexnet_tencrop(alexnet_t* h, const uint8_t* src, int B, const float* mean,
                               float* probs_avg, int32_t* top5, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!src || !mean || !probs_avg || !top5 || B < 1) {
    h->err = "tencrop: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  if (h->cfg.dtype != ALEXNET_BF16) {
    h->err = "tencrop: bf16 handles only";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  const int chunk = h->cfg.batch_max / 10;
  if (chunk < 1) {
    h->err = "tencrop: batch_max must be >= 10";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  write_hp(h, 0.f, s);
  for (int b0 = 0; b0 < B; b0 += chunk) {
    const int nb = B - b0 < chunk ? B - b0 : chunk;
    Plan* P = get_plan(h, nb * 10);
    if (!P) return ALEXNET_ERR_CUDA;
    launch_tencrop_inputs(src + static_cast<size_t>(b0) * 256 * 256 * 3, nb, mean, h->xin, s);
    alexnet_status st = forward_bf16(h, h->xin, nb * 10, h->cfg.dropout_on ? 2 : 0, h->logits, s, P);
    if (st != ALEXNET_OK) return st;
    launch_softmax_ce(h->logits, nullptr, nb * 10, kClasses, h->probs, nullptr, nullptr, h->status,
                      s);
    launch_tencrop_reduce(h->probs, nb, kClasses, probs_avg + static_cast<size_t>(b0) * kClasses,
                          top5 + static_cast<size_t>(b0) * 5, s);
  }
  return cuda_status(h, cudaGetLastError(), "tencrop");
}

size_t alexnet_ensemble_workspace_bytes(int n_models, int B) {
  if (n_models < 1 || B < 1) return 0;
  return (static_cast<size_t>(n_models) + 1) * B * kClasses * sizeof(float);
}

alexnet_status alexnet_ensemble_forward(alexnet_t* const* nets, int n_models, const void* x,
                                        int B, float* probs_avg, int32_t* top5, void* ws,
                                        size_t ws_bytes, void* stream) {
  if (!nets || n_models < 1 || !x || B < 1 || !probs_avg || !top5 || !ws ||
      ws_bytes < alexnet_ensemble_workspace_bytes(n_models, B))
    return ALEXNET_ERR_INVALID_ARG;
  for (int m = 0; m < n_models; ++m)
    if (!nets[m] || nets[m]->cfg.dtype != nets[0]->cfg.dtype || B > nets[m]->cfg.batch_max)
      return ALEXNET_ERR_INVALID_ARG;
  float* logits = static_cast<float*>(ws);
  float* probs = logits + static_cast<size_t>(B) * kClasses;
  for (int m = 0; m < n_models; ++m) {
    const alexnet_status st =
        alexnet_forward(nets[m], x, B, ALEXNET_INFERENCE, logits,
                        probs + static_cast<size_t>(m) * B * kClasses, stream);
    if (st != ALEXNET_OK) return st;
  }
  launch_ensemble_reduce(probs, n_models, B, kClasses, probs_avg, top5,
                         static_cast<cudaStream_t>(stream));
  return cudaGetLastError() == cudaSuccess ? ALEXNET_OK : ALEXNET_ERR_CUDA;
}

size_t alexnet_params_bytes(const alexnet_t* h) {
  return h ? 8 * h->n_params + 8 : 0;
}

alexnet_status alexnet_get_params(alexnet_t* h, void* dst, size_t bytes, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!dst || bytes < alexnet_params_bytes(h)) {
    h->err = "get_params: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  ALX_TRY(cudaMemcpyAsync(dst, h->params, 8 * h->n_params, cudaMemcpyDefault, s), "get_params");
  ALX_TRY(cudaMemcpyAsync(static_cast<char*>(dst) + 8 * h->n_params, &h->step, 8,
                          cudaMemcpyDefault, s),
          "get_params");
  ALX_TRY(cudaStreamSynchronize(s), "get_params");
  return ALEXNET_OK;
}

alexnet_status alexnet_set_params(alexnet_t* h, const void* src, size_t bytes, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!src || bytes < alexnet_params_bytes(h)) {
    h->err = "set_params: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  h->last_stream = s;
  ALX_TRY(cudaMemcpyAsync(h->params, src, 8 * h->n_params, cudaMemcpyDefault, s), "set_params");
  uint64_t step = 0;
  ALX_TRY(cudaMemcpyAsync(&step, static_cast<const char*>(src) + 8 * h->n_params, 8,
                          cudaMemcpyDefault, s),
          "set_params");
  ALX_TRY(cudaStreamSynchronize(s), "set_params");
  h->step = step;
  refresh_shadows(h, s);
  return cuda_status(h, cudaGetLastError(), "set_params");
}

alexnet_status alexnet_get_grads(alexnet_t* h, float* dst, size_t n, void* stream) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  if (!h->grads) {
    h->err = "get_grads: handle was created without keep_grads";
    return ALEXNET_ERR_UNSUPPORTED;
  }
  if (!dst || n < h->n_params) {
    h->err = "get_grads: invalid argument";
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ALX_TRY(cudaMemcpyAsync(dst, h->grads, 4 * h->n_params, cudaMemcpyDefault, s), "get_grads");
  ALX_TRY(cudaStreamSynchronize(s), "get_grads");
  return ALEXNET_OK;
}

alexnet_status alexnet_get_status(alexnet_t* h) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e != cudaSuccess) return cuda_status(h, e, "get_status");
  int st = 0;
  e = cudaMemcpy(&st, h->status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(h, e, "get_status");
  if (st & STATUS_TIMEOUT) {
    h->err = "a device wait ran out of time";
    return ALEXNET_ERR_TIMEOUT;
  }
  if (st & STATUS_LABEL_RANGE) {
    h->err = "a label was outside [0, 1000)";
    return ALEXNET_ERR_LABEL_RANGE;
  }
  return ALEXNET_OK;
}

const char* alexnet_last_error(const alexnet_t* h) {
  return h ? h->err.c_str() : g_create_error.c_str();
}

alexnet_status alexnet_destroy(alexnet_t* h) {
  if (h) {
    for (cudaEvent_t e : h->direct_rec.ev) cudaEventDestroy(e);
    for (auto& kv : h->graph_rec)
      for (cudaEvent_t e : kv.second.ev) cudaEventDestroy(e);
    for (auto& kv : h->train_graphs) cudaGraphExecDestroy(kv.second);
    if (h->fc_event) cudaEventDestroy(h->fc_event);
    if (h->cap_stream) cudaStreamDestroy(h->cap_stream);
    if (h->side) cudaStreamDestroy(h->side);
    for (int l = 0; l < 5; ++l) {
      if (h->ev_dy[l]) cudaEventDestroy(h->ev_dy[l]);
      if (h->ev_dg[l]) cudaEventDestroy(h->ev_dg[l]);
    }
    for (int f = 0; f < 3; ++f) {
      if (h->ev_fdz[f]) cudaEventDestroy(h->ev_fdz[f]);
      if (h->ev_fdg[f]) cudaEventDestroy(h->ev_fdg[f]);
    }
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->ev_fjoin) cudaEventDestroy(h->ev_fjoin);
  }
  delete h;
  return ALEXNET_OK;
}

alexnet_status alexnet_stats_enable(alexnet_t* h, int enable) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  h->stats_on = enable != 0;
  h->last_rec = nullptr;
  h->last_launches = 0;
  return ALEXNET_OK;
}

alexnet_status alexnet_conv_algo(alexnet_t* h, int batch, int layer, int pass, int* algo) {
  if (!h || !algo || layer < 0 || layer > 4 || pass < 0 || pass > 2 || (pass == 1 && layer == 0) ||
      batch < 1 || batch > h->cfg.batch_max || h->cfg.dtype != ALEXNET_BF16)
    return ALEXNET_ERR_INVALID_ARG;
  Plan* P = get_plan(h, batch);
  if (!P) return ALEXNET_ERR_UNSUPPORTED;
  const ConvPlan& c = pass == 0 ? P->cf[layer] : (pass == 1 ? P->cd[layer] : P->cw[layer]);
  *algo = c.box ? 1 : 0;
  return ALEXNET_OK;
}

alexnet_status alexnet_debug_keep(alexnet_t* h, int keep) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  h->keep = keep != 0;
  return ALEXNET_OK;
}

alexnet_status alexnet_debug_fc_update(alexnet_t* h, int fused) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  h->fc_fused = fused != 0;
  return ALEXNET_OK;
}

alexnet_status alexnet_debug_overlap(alexnet_t* h, int on) {
  if (!h) return ALEXNET_ERR_INVALID_ARG;
  h->overlap_wgrad = on != 0;
  return ALEXNET_OK;
}

alexnet_status alexnet_stats_read(alexnet_t* h, alexnet_stats* out) {
  if (!h || !out) return ALEXNET_ERR_INVALID_ARG;
  memset(out, 0, sizeof(*out));
  if (!h->last_rec) return ALEXNET_OK;
  ALX_TRY(cudaStreamSynchronize(h->stats_stream), "stats_read");
  double ms = 0.0;
  const alexnet::StepRec& R = *h->last_rec;
  for (size_t i = 0; i + 1 < R.used; i += 2) {
    float t = 0.f;
    ALX_TRY(cudaEventElapsedTime(&t, R.ev[i], R.ev[i + 1]), "stats_read");
    ms += t;
  }
  out->launches = h->last_launches;
  out->gemm_launches = R.gemm_launches;
  out->gemm_flops = R.gemm_flops;
  out->gemm_ms = ms;
  return ALEXNET_OK;
}

alexnet_status alexnet_stats_launch(alexnet_t* h, int i, int* kind, double* flops, double* ms) {
  if (!h || !kind || !flops || !ms || i < 0) return ALEXNET_ERR_INVALID_ARG;
  if (!h->last_rec || static_cast<size_t>(i) >= h->last_rec->flops.size())
    return ALEXNET_ERR_INVALID_ARG;
  ALX_TRY(cudaStreamSynchronize(h->stats_stream), "stats_launch");
  const alexnet::StepRec& R = *h->last_rec;
  float t = 0.f;
  ALX_TRY(cudaEventElapsedTime(&t, R.ev[2 * i], R.ev[2 * i + 1]), "stats_launch");
  *kind = R.kind[i];
  *flops = R.flops[i];
  *ms = t;
  return ALEXNET_OK;
}

alexnet_status alexnet_debug_canaries(alexnet_t* h, int64_t* bad_bytes) {
  if (!h || !bad_bytes) return ALEXNET_ERR_INVALID_ARG;
  *bad_bytes = 0;
  cudaError_t e = cudaStreamSynchronize(h->last_stream);
  if (e != cudaSuccess) return cuda_status(h, e, "debug_canaries");
  std::vector<unsigned char> buf(kCanaryBytes);
  int64_t bad = 0;
  for (size_t g : h->guards) {
    e = cudaMemcpy(buf.data(), h->ws + g, kCanaryBytes, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(h, e, "debug_canaries");
    for (unsigned char b : buf) bad += b != kCanaryByte;
  }
  *bad_bytes = bad;
  return ALEXNET_OK;
}

alexnet_status alexnet_debug_copy(alexnet_t* h, int which, void* dst, size_t bytes, void* stream) {
  if (!h || !dst) return ALEXNET_ERR_INVALID_ARG;
  if (h->cfg.dtype != ALEXNET_BF16) return ALEXNET_ERR_UNSUPPORTED;
  const int B = h->cfg.batch_max;
  const void* src = nullptr;
  size_t n = 0;
  if (which >= 0 && which < 5) {
    const ConvL& L = h->conv[which];
    src = h->a[which];
    n = 2ull * B * L.Ho * L.Ho * L.Cout;
  } else if ((which == 10 || which == 11) && h->lo[which - 10]) {
    const ConvL& L = h->conv[which - 10];
    src = h->lo[which - 10];
    n = 2ull * B * L.Ho * L.Ho * L.Cout;
  } else if ((which == 20 || which == 21 || which == 24) && h->p[which - 20]) {
    const ConvL& L = h->conv[which - 20];
    src = h->p[which - 20];
    n = 2ull * B * L.P * L.P * L.Cout;
  } else if (which == 30 || which == 31) {
    src = which == 30 ? h->f6 : h->f7;
    n = 2ull * B * 4096;
  } else if (which == 40) {
    src = h->logits;
    n = 4ull * B * kClasses;
  } else if (which >= 50 && which < 55) {
    const ConvL& L = h->conv[which - 50];
    src = h->da[which - 50];
    n = 2ull * B * L.Ho * L.Ho * L.Cout;
  } else if (which >= 60 && which < 65 && h->dp[which - 60]) {
    const ConvL& L = h->conv[which - 60];
    src = h->dp[which - 60];
    n = 2ull * B * L.P * L.P * L.Cout;
  } else if (which >= 70 && which < 75 && h->dl[which - 70]) {
    const ConvL& L = h->conv[which - 70];
    src = h->dl[which - 70];
    n = 2ull * B * L.Ho * L.Ho * L.Cout;
  } else if (which == 80) {
    src = h->dlogits;
    n = 2ull * B * kClasses;
  } else if (which == 81 || which == 82) {
    src = which == 81 ? h->d7 : h->d6;
    n = 2ull * B * 4096;
  } else if ((which == 90 || which == 91 || which == 94) && h->am[which - 90]) {
    const ConvL& L = h->conv[which - 90];
    src = h->am[which - 90];
    n = 1ull * B * L.P * L.P * L.Cout;
  } else {
    return ALEXNET_ERR_INVALID_ARG;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  ALX_TRY(cudaMemcpyAsync(dst, src, bytes < n ? bytes : n, cudaMemcpyDefault, s), "debug_copy");
  return ALEXNET_OK;
}

}  // extern "C"
