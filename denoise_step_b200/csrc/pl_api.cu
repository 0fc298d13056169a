// C ABI (include/pl.h): argument validation, workspace layout, launch order
// of one round and its CUDA-graph capture.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/pl.h"
#include "attn.cuh"
#include "devinit.cuh"
#include "gemm.cuh"
#include "misc.cuh"
#include "ptx.cuh"

using pl::AttnParams;
using pl::AttnSegHost;
using pl::GemmParams;

namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxSessions = 8;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int num_sms() { return pl::device_sms(); }

bool head_dim_supported(int hd) {
  return hd == 40 || hd == 64 || hd == 80 || hd == 128 || hd == 160;
}

pl_status from_cuda(cudaError_t e) { return e == cudaSuccess ? PL_OK : PL_ECUDA; }

pl_status gemm_status(int r) {
  return r == 0 ? PL_OK : r == 1 ? PL_EINVAL : r == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
}

// Status word of the calls made without a context (one per device that uses
// the library): kernels OR their device-side problems into it, and
// pl_get_call_status() reads and clears it.
static __device__ uint32_t g_call_status;

std::mutex g_dev_mu;
uint32_t* g_call_status_ptr[pl::kMaxDevices] = {};
int g_sms[pl::kMaxDevices] = {};

}  // namespace

namespace pl {

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

uint32_t* call_status_word() {
  const int dev = current_device();
  if (dev < 0) return nullptr;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (!g_call_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_call_status) != cudaSuccess) return nullptr;
    g_call_status_ptr[dev] = static_cast<uint32_t*>(p);
  }
  return g_call_status_ptr[dev];
}

int device_sms() {
  const int dev = current_device();
  if (dev < 0) return 148;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  if (g_sms[dev] <= 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sms[dev] = n;
  }
  return g_sms[dev];
}

}  // namespace pl


// ====================================================================== context

// streams one round's layers are spread over (inside its captured graph).
// Measured on the 512x512 round (same box, three runs each): one stream
// 19.68-19.87 ms, two 19.38-19.49 ms, three 19.34-19.44 ms, four 19.25-19.37
// ms; each stream beyond the first holds its own layer scratch (~340 MB per
// session at 512x512), so two.
constexpr int kRoundStreams = 2;
static_assert(kRoundStreams >= 2, "the fork and join expect a second stream");

struct pl_ctx {
  pl_config cfg;
  int sessions;        // S independent streams; per-stream buffers are [S][...]
  int capacity;        // motion/KV bank capacity = 1 + append_cap
  int64_t frame_elems; // latent_c * H * W
  uint8_t* ws;
  size_t ws_bytes;
  pl::DevState* st;    // [S]
  float* ring;
  float* slot_motion;
  float* batch_motion;
  float* bank;
  int motion_blocks;   // motion cross-attention blocks per layer (1 or 2)
  __half* bank_kv[PL_MAX_LAYERS];     // fp16 [S][capacity][N][2C]
  float* motion_kv[PL_MAX_LAYERS];   // fp32 [S][16][32][2C]
  float* motion_kv2[PL_MAX_LAYERS];  // second motion block's, as motion_kv
  __half* w_oq[PL_MAX_LAYERS];        // fp16 [C][C] = Wo Mq
  __half* w_oq2[PL_MAX_LAYERS];       // fp16 [C][C] = Mo Mq2 (two motion blocks)
  // per-layer scratch, one set per round stream: layer l runs on stream
  // l % kRoundStreams with set l % kRoundStreams (the layers are independent:
  // each has its own hidden input and output)
  struct Scratch {
    __half* qkv;
    __half* attn_o;
    __half* a1;
    float* qm;          // fp32 motion queries (Mq accumulators); on the folded
                        // path the fp16 probabilities P [M][32 H]
    __half* om;
    __half* out_default;
    __half* fold_wqk;   // folded motion path: fp16 [S][16][C][32 H]
    __half* fold_vm;    // and fp16 [S][16][32 H][C]
  } sc[kRoundStreams];
  cudaStream_t side[kRoundStreams - 1];   // the round's other streams
  cudaEvent_t ev_fork;                    // their fork after the ring push
  cudaEvent_t ev_join[kRoundStreams - 1];  // and their joins
  pl::DdimCoef coef;
  bool initialised;
  bool have_anchors;
  pl_layer_weights w[PL_MAX_LAYERS];
  const void* ref_feats[PL_MAX_LAYERS];
  const void* anchor_feats[3][PL_MAX_LAYERS];
  // captured rounds, one per pointer set (two: the host path alternates
  // between its staging sets)
  struct GraphSlot {
    cudaGraph_t graph;
    cudaGraphExec_t exec;
    const void* key[64];
    int key_n;
    int kernels;            // kernel nodes of the captured round
    uint64_t last_use;
  } graphs[2];
  uint64_t graph_tick;
  int last_round_kernels;   // kernels of the last round run from a capture (-1: none)
  // host path: copy stream, staging-set events, rounds issued
  cudaStream_t copy_stream;
  cudaEvent_t ev_in[2];     // set b's inputs are on the device
  cudaEvent_t ev_free[2];   // the round reading set b is done
  bool free_pending[2];
  int64_t host_rounds;
  // per-layer timing of rounds run outside the captured graph
  bool profile;
  bool prof_valid;             // the events hold a finished profiled round
  cudaEvent_t prof_ev[PL_MAX_LAYERS + 1];
};

namespace {

// The motion cross-attention runs folded (scores X W_qk with the softmax in
// the GEMM epilogue, output P VM) on layers of at least this many tokens per
// frame. Measured on the 512x512 round (graph-captured, same box, three runs
// each): 20.12 ms unfolded, 19.75 ms folded at 64x64; with the fold kernel
// reading eight head channels per step, 19.84 ms folded at 64x64 against
// 19.74 ms at 32x32 too (its layers 0.501 -> 0.475 ms). At 16x16 and below
// forming W_qk and VM (which grows with C^2) costs more than the attention.
constexpr int kFoldMinTokens = 1024;
bool fold_layer(const pl_config& c, int l) {
  return c.layer_tokens[l] >= kFoldMinTokens && 16 * c.heads <= c.layer_channels[l];
}

// Workspace layout; with ctx == nullptr only the size is computed.
size_t layout(const pl_config& c, pl_ctx* ctx) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> uint8_t* {
    uint8_t* p = ctx ? ctx->ws + off : nullptr;
    off += align_up(bytes);
    return p;
  };
  const int capacity = 1 + c.append_cap;
  const int64_t S = c.sessions > 0 ? c.sessions : 1;
  const bool two = c.motion_blocks == 2;
  const int64_t fe = static_cast<int64_t>(c.latent_c) * c.latent_h * c.latent_w;
  uint8_t* st = take(sizeof(pl::DevState) * S);
  uint8_t* ring = take(sizeof(float) * S * 16 * fe);
  uint8_t* sm = take(sizeof(float) * S * 16 * 512);
  uint8_t* bm = take(sizeof(float) * S * 16 * 512);
  uint8_t* bank = take(sizeof(float) * S * capacity * 512);
  int64_t max_nc = 0;
  for (int l = 0; l < c.n_layers; ++l) {
    const int64_t N = c.layer_tokens[l], C = c.layer_channels[l];
    uint8_t* bkv = take(sizeof(__half) * S * capacity * N * 2 * C);
    uint8_t* mkv = take(sizeof(float) * S * 16 * 32 * 2 * C);
    uint8_t* mkv2 = two ? take(sizeof(float) * S * 16 * 32 * 2 * C) : nullptr;
    uint8_t* woq = take(sizeof(__half) * C * C);
    uint8_t* woq2 = two ? take(sizeof(__half) * C * C) : nullptr;
    if (ctx) {
      ctx->bank_kv[l] = reinterpret_cast<__half*>(bkv);
      ctx->motion_kv[l] = reinterpret_cast<float*>(mkv);
      ctx->motion_kv2[l] = reinterpret_cast<float*>(mkv2);
      ctx->w_oq[l] = reinterpret_cast<__half*>(woq);
      ctx->w_oq2[l] = reinterpret_cast<__half*>(woq2);
    }
    if (S * 16 * N * C > max_nc) max_nc = S * 16 * N * C;
  }
  int64_t fold_c = 0;
  for (int l = 0; l < c.n_layers; ++l)
    if (fold_layer(c, l) && c.layer_channels[l] > fold_c) fold_c = c.layer_channels[l];
  const int64_t fold_elems = S * 16 * fold_c * 32 * c.heads;
  for (int k = 0; k < kRoundStreams; ++k) {
    uint8_t* qkv = take(sizeof(__half) * 3 * max_nc);
    uint8_t* ao = take(sizeof(__half) * max_nc);
    uint8_t* a1 = take(sizeof(__half) * max_nc);
    uint8_t* qm = take(sizeof(float) * max_nc);
    uint8_t* om = take(sizeof(__half) * max_nc);
    uint8_t* od = take(sizeof(__half) * max_nc);
    uint8_t* fwqk = fold_elems ? take(sizeof(__half) * fold_elems) : nullptr;
    uint8_t* fvm = fold_elems ? take(sizeof(__half) * fold_elems) : nullptr;
    if (ctx) {
      pl_ctx::Scratch& x = ctx->sc[k];
      x.qkv = reinterpret_cast<__half*>(qkv);
      x.attn_o = reinterpret_cast<__half*>(ao);
      x.a1 = reinterpret_cast<__half*>(a1);
      x.qm = reinterpret_cast<float*>(qm);
      x.om = reinterpret_cast<__half*>(om);
      x.out_default = reinterpret_cast<__half*>(od);
      x.fold_wqk = reinterpret_cast<__half*>(fwqk);
      x.fold_vm = reinterpret_cast<__half*>(fvm);
    }
  }
  if (ctx) {
    ctx->st = reinterpret_cast<pl::DevState*>(st);
    ctx->ring = reinterpret_cast<float*>(ring);
    ctx->slot_motion = reinterpret_cast<float*>(sm);
    ctx->batch_motion = reinterpret_cast<float*>(bm);
    ctx->bank = reinterpret_cast<float*>(bank);
  }
  return off;
}

pl_status validate_config(const pl_config* c) {
  if (!c) return PL_EINVAL;
  if (c->latent_c < 1 || c->latent_h < 1 || c->latent_w < 1) return PL_EINVAL;
  if ((static_cast<int64_t>(c->latent_c) * c->latent_h * c->latent_w) % 4) return PL_EINVAL;
  if (c->n_layers < 0 || c->n_layers > PL_MAX_LAYERS) return PL_EINVAL;
  if (c->heads < 1) return PL_EINVAL;
  if (c->append_cap < 0 || c->append_cap > PL_MAX_BANK - 1) return PL_EINVAL;
  if (!(c->drift_threshold >= 0.f) || !std::isfinite(c->drift_threshold)) return PL_EINVAL;
  if (c->sessions < 0 || c->sessions > kMaxSessions) return PL_EINVAL;
  if (c->motion_blocks < 0 || c->motion_blocks > 2) return PL_EINVAL;
  for (int l = 0; l < c->n_layers; ++l) {
    const int N = c->layer_tokens[l], C = c->layer_channels[l];
    if (N < 1 || C < 1 || C % c->heads || C % 16) return PL_EINVAL;
    if (!head_dim_supported(C / c->heads)) return PL_EUNSUPPORTED;
  }
  return PL_OK;
}

// Grouped K/V projection of bank features (device fp16 [S][N_l][C_l] per
// layer) into entry `entry` of every layer, one grouped launch per session;
// with `predicated` a session's launch only runs when that session's bank
// check appended anchor `entry` this round.
pl_status project_bank(pl_ctx* ctx, const void* const* feats, int entry, bool predicated,
                       cudaStream_t s, int only_session = -1) {
  for (int z = 0; z < ctx->sessions; ++z) {
    if (only_session >= 0 && z != only_session) continue;
    GemmParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.status = &ctx->st[z].status;
    const int32_t* pred = predicated ? &ctx->st[z].anchor_fire[entry] : nullptr;
    int np = 0;
    for (int l = 0; l < ctx->cfg.n_layers; ++l) {
      if (!feats[l]) return PL_EINVAL;
      const int64_t N = ctx->cfg.layer_tokens[l], C = ctx->cfg.layer_channels[l];
      const __half* wkv = static_cast<const __half*>(ctx->w[l].w_qkv) + C;
      const __half* a = static_cast<const __half*>(feats[l]) + z * N * C;
      __half* dst = ctx->bank_kv[l] + (static_cast<int64_t>(z) * ctx->capacity + entry) * N * 2 * C;
      const int r = pl::gemm_make_problem(&gp.prob[np], a, C, wkv, 3 * C, dst, 2 * C,
                                          static_cast<int>(N), static_cast<int>(2 * C),
                                          static_cast<int>(C), pred);
      if (r) return gemm_status(r);
      ++np;
    }
    gp.n_problems = np;
    if (np == 0) return PL_OK;
    const pl_status r = gemm_status(pl::gemm_launch(&gp, s, num_sms()));
    if (r) return r;
  }
  return PL_OK;
}

pl_status single_gemm(const void* a, int64_t lda, const void* b, int64_t ldb, void* c,
                      int64_t ldc, int M, int N, int K, uint32_t* status, cudaStream_t s,
                      bool out_f32 = false) {
  GemmParams gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.status = status;
  const int r =
      pl::gemm_make_problem(&gp.prob[0], a, lda, b, ldb, c, ldc, M, N, K, nullptr, out_f32);
  if (r) return gemm_status(r);
  gp.n_problems = 1;
  return gemm_status(pl::gemm_launch(&gp, s, num_sms()));
}

// One GEMM per frame f < F with a B of its own: C_f = A_f B_f, where A_f =
// a + f N lda, B_f = b + f b_stride and C_f = c + f N ldc hold N rows each;
// up to kGemmMaxProblems frames per launch. softmax32: fp16 output with each
// 32-column group replaced by its softmax (base-2 logits).
pl_status frame_gemm(const __half* a, int64_t lda, const __half* b, int64_t ldb, int64_t b_stride,
                     __half* c, int64_t ldc, int F, int N, int n_cols, int K, bool softmax32,
                     uint32_t* status, cudaStream_t s) {
  for (int f0 = 0; f0 < F; f0 += pl::kGemmMaxProblems) {
    GemmParams gp;
    std::memset(&gp, 0, sizeof(gp));
    gp.status = status;
    const int nf = F - f0 < pl::kGemmMaxProblems ? F - f0 : pl::kGemmMaxProblems;
    for (int i = 0; i < nf; ++i) {
      const int64_t f = f0 + i;
      const int r = pl::gemm_make_problem(&gp.prob[i], a + f * N * lda, lda, b + f * b_stride, ldb,
                                          c + f * N * ldc, ldc, N, n_cols, K, nullptr, false);
      if (r) return gemm_status(r);
      if (softmax32 && pl::gemm_set_softmax32(&gp.prob[i])) return PL_EINVAL;
    }
    gp.n_problems = nf;
    const pl_status r = gemm_status(pl::gemm_launch(&gp, s, num_sms()));
    if (r) return r;
  }
  return PL_OK;
}

struct RoundArgs {
  const float* new_noise;
  const float* new_motion;
  const void* const* hidden;
  const float* eps;
  float* out_frames;
  uint8_t* appended;
  void* const* layer_out;
  void* const* attn_out;
  cudaEvent_t* layer_events;   // when non-null: [n_layers + 1] recorded around the layers
};

// Enqueue layer l of a round on `s` with scratch set `sc`.
pl_status enqueue_layer(pl_ctx* ctx, const RoundArgs& a, int l, const pl_ctx::Scratch& sc,
                        cudaStream_t s) {
  const pl_config& c = ctx->cfg;
  const int S = ctx->sessions;
  const int F = 16 * S;   // the batches of all sessions, session-major
  pl_status r = PL_OK;
  const int N = c.layer_tokens[l], C = c.layer_channels[l], H = c.heads, hd = C / H;
  const int64_t M = static_cast<int64_t>(F) * N;
  const pl_layer_weights& w = ctx->w[l];
  __half* out = a.layer_out ? static_cast<__half*>(a.layer_out[l]) : sc.out_default;
  r = from_cuda(pl::launch_motion_kv(ctx->batch_motion, static_cast<const __half*>(w.m_kv), F,
                                     C, ctx->motion_kv[l], s));
  if (r) return r;
  if (ctx->motion_blocks == 2) {
    r = from_cuda(pl::launch_motion_kv(ctx->batch_motion, static_cast<const __half*>(w.m2_kv),
                                       F, C, ctx->motion_kv2[l], s));
    if (r) return r;
  }
  r = single_gemm(a.hidden[l], C, w.w_qkv, 3 * C, sc.qkv, 3 * C, static_cast<int>(M), 3 * C,
                  C, &ctx->st->status, s);
  if (r) return r;
  // own K/V per frame; bank entry b of session z for the frames of session z
  AttnSegHost segs[1 + PL_MAX_BANK];
  segs[0] = {sc.qkv + C, sc.qkv + 2 * C, N, 3ll * C, static_cast<int64_t>(N) * 3 * C};
  const int nb = ctx->have_anchors ? ctx->capacity : 1;
  for (int b = 0; b < nb; ++b) {
    const __half* kv = ctx->bank_kv[l] + static_cast<int64_t>(b) * N * 2 * C;
    segs[1 + b] = {kv, kv + C, N, 2ll * C, 0};
    if (S > 1) {
      segs[1 + b].frame_stride = static_cast<int64_t>(ctx->capacity) * N * 2 * C;
      segs[1 + b].n_blocks = S;
      segs[1 + b].frame_div = 16;
    }
  }
  AttnParams ap;
  int ar = pl::attn_make_params(&ap, sc.qkv, 3ll * C, static_cast<int64_t>(N) * 3 * C, segs,
                                1 + nb, F, N, H, hd, sc.attn_o, C,
                                static_cast<int64_t>(N) * C);
  if (ar) return ar == 1 ? PL_EINVAL : PL_ECUDA;
  ap.n_fixed = 2;
  ap.n_extra = ctx->have_anchors ? &ctx->st->appends : nullptr;
  ap.extra_div = 16;
  ap.extra_stride = static_cast<int>(sizeof(pl::DevState) / sizeof(int32_t));
  ap.status = &ctx->st->status;
  ar = pl::attn_launch(ap, hd, s);
  if (ar) return ar == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
  uint32_t* status = &ctx->st->status;
  const int Mi = static_cast<int>(M);
  if (fold_layer(c, l)) {
    // motion cross-attention, folded: per frame the scores X W_qk with the
    // softmax over each head's 32 tokens in the GEMM epilogue (P, fp16, in
    // the query buffer), then the block output P VM; block 2 takes block 1's
    // output as its X
    const int NT = 32 * H;
    __half* P = reinterpret_cast<__half*>(sc.qm);
    const __half* x = sc.attn_o;
    const void* wq = ctx->w_oq[l];   // O (Wo Mq)
    if (a.attn_out) {
      // the sub-layer output is wanted: O Wo, then its motion queries
      __half* a1 = static_cast<__half*>(a.attn_out[l]);
      r = single_gemm(sc.attn_o, C, w.w_o, C, a1, C, Mi, C, C, status, s);
      if (r) return r;
      x = a1;
      wq = w.m_q;
    }
    for (int b = 0; b < ctx->motion_blocks; ++b) {
      const bool second = b == 1;
      __half* y = b == ctx->motion_blocks - 1 ? out : sc.om;
      r = from_cuda(pl::launch_motion_fold(
          second ? ctx->motion_kv2[l] : ctx->motion_kv[l],
          static_cast<const __half*>(second ? w.m2_q : wq),
          static_cast<const __half*>(second ? w.m2_o : w.m_o), F, C, H, sc.fold_wqk,
          sc.fold_vm, s));
      if (r) return r;
      r = frame_gemm(x, C, sc.fold_wqk, NT, static_cast<int64_t>(C) * NT, P, NT, F, N, NT, C,
                     true, status, s);
      if (r) return r;
      r = frame_gemm(P, NT, sc.fold_vm, C, static_cast<int64_t>(NT) * C, y, C, F, N, C, NT,
                     false, status, s);
      if (r) return r;
      x = y;
    }
  } else {
    if (a.attn_out) {
      // the sub-layer output is wanted: O Wo, then its motion queries
      __half* a1 = static_cast<__half*>(a.attn_out[l]);
      r = single_gemm(sc.attn_o, C, w.w_o, C, a1, C, Mi, C, C, status, s);
      if (r) return r;
      r = single_gemm(a1, C, w.m_q, C, sc.qm, C, Mi, C, C, status, s, /*out_f32=*/true);
    } else {
      // motion queries straight from O: O (Wo Mq)
      r = single_gemm(sc.attn_o, C, ctx->w_oq[l], C, sc.qm, C, Mi, C, C, status, s,
                      /*out_f32=*/true);
    }
    if (r) return r;
    r = from_cuda(
        pl::launch_motion_attn(sc.qm, C, ctx->motion_kv[l], F, N, C, H, sc.om, C, s));
    if (r) return r;
    if (ctx->motion_blocks == 2) {
      // block 2's queries from block 1's output: y1 Mq2 = om (Mo Mq2)
      if (a.attn_out) {
        r = single_gemm(sc.om, C, w.m_o, C, sc.a1, C, Mi, C, C, status, s);
        if (r) return r;
        r = single_gemm(sc.a1, C, w.m2_q, C, sc.qm, C, Mi, C, C, status, s, true);
      } else {
        r = single_gemm(sc.om, C, ctx->w_oq2[l], C, sc.qm, C, Mi, C, C, status, s, true);
      }
      if (r) return r;
      r = from_cuda(pl::launch_motion_attn(sc.qm, C, ctx->motion_kv2[l], F, N, C, H, sc.om,
                                           C, s));
      if (r) return r;
    }
    const void* w_last = ctx->motion_blocks == 2 ? w.m2_o : w.m_o;
    r = single_gemm(sc.om, C, w_last, C, out, C, Mi, C, C, status, s);
    if (r) return r;
  }
  return PL_OK;
}

// Enqueue one whole round on `s` (also used under stream capture).
pl_status enqueue_round(pl_ctx* ctx, const RoundArgs& a, cudaStream_t s) {
  const pl_config& c = ctx->cfg;
  const int S = ctx->sessions;
  const int F = 16 * S;   // the batches of all sessions, session-major
  pl_status r = from_cuda(pl::launch_ring_push(ctx->st, ctx->ring, ctx->slot_motion,
                                               ctx->batch_motion, a.new_noise, a.new_motion,
                                               ctx->frame_elems, S, s));
  if (r) return r;
  // layers are independent (each has its own hidden input and output):
  // layer l runs on round stream l % kRoundStreams with its scratch set, the
  // other streams forked after the ring push (motion K/V read its batch
  // motion) and joined before the DDIM step and the bank check (its appends
  // change the bank length the attention reads). Profiled rounds keep one
  // stream so that the layer events bracket layers.
  const bool fork = !a.layer_events && kRoundStreams > 1 && ctx->side[0] != nullptr &&
                    c.n_layers > 1;
  if (fork) {
    if (cudaEventRecord(ctx->ev_fork, s) != cudaSuccess) return PL_ECUDA;
    for (int k = 0; k + 1 < kRoundStreams; ++k)
      if (cudaStreamWaitEvent(ctx->side[k], ctx->ev_fork, 0) != cudaSuccess) return PL_ECUDA;
  }
  for (int l = 0; l < c.n_layers && r == PL_OK; ++l) {
    if (a.layer_events && cudaEventRecord(a.layer_events[l], s) != cudaSuccess) {
      r = PL_ECUDA;
      break;
    }
    const int k = fork ? l % kRoundStreams : 0;
    r = enqueue_layer(ctx, a, l, ctx->sc[k], k ? ctx->side[k - 1] : s);
  }
  // the joins also close the fork after a failure, so a capture can end
  if (fork)
    for (int k = 0; k + 1 < kRoundStreams; ++k)
      if (cudaEventRecord(ctx->ev_join[k], ctx->side[k]) != cudaSuccess ||
          cudaStreamWaitEvent(s, ctx->ev_join[k], 0) != cudaSuccess)
        return PL_ECUDA;
  if (r) return r;
  if (a.layer_events && c.n_layers > 0 &&
      cudaEventRecord(a.layer_events[c.n_layers], s) != cudaSuccess)
    return PL_ECUDA;
  r = from_cuda(pl::launch_ddim(ctx->st, ctx->ring, a.eps, a.out_frames, ctx->frame_elems,
                                ctx->coef, S, s));
  if (r) return r;
  r = from_cuda(pl::launch_ring_commit(ctx->st, S, s));
  if (r) return r;
  r = from_cuda(pl::launch_bank_check(ctx->bank, nullptr, nullptr, ctx->capacity, 512,
                                      a.new_motion, 4,
                                      static_cast<double>(c.drift_threshold) * c.drift_threshold,
                                      c.append_cap, nullptr, nullptr, a.appended, ctx->st, S,
                                      nullptr, s));
  if (r) return r;
  if (ctx->have_anchors) {
    for (int an = 1; an <= c.append_cap; ++an) {
      r = project_bank(ctx, ctx->anchor_feats[an - 1], an, /*predicated=*/true, s);
      if (r) return r;
    }
  }
  return PL_OK;
}

void drop_slot(pl_ctx::GraphSlot& g) {
  if (g.exec) cudaGraphExecDestroy(g.exec);
  if (g.graph) cudaGraphDestroy(g.graph);
  g.exec = nullptr;
  g.graph = nullptr;
  g.key_n = 0;
  g.kernels = 0;
}

// kernel nodes of a captured graph (-1 when the graph cannot be read)
int count_kernel_nodes(cudaGraph_t g) {
  size_t n = 0;
  if (cudaGraphGetNodes(g, nullptr, &n) != cudaSuccess) return -1;
  std::vector<cudaGraphNode_t> nodes(n);
  if (n && cudaGraphGetNodes(g, nodes.data(), &n) != cudaSuccess) return -1;
  int k = 0;
  for (size_t i = 0; i < n; ++i) {
    cudaGraphNodeType t;
    if (cudaGraphNodeGetType(nodes[i], &t) != cudaSuccess) return -1;
    if (t == cudaGraphNodeTypeKernel) ++k;
  }
  return k;
}

void drop_graph(pl_ctx* ctx) {
  for (auto& g : ctx->graphs) drop_slot(g);
}

// Staging of the host path: two sets, each the inputs of one round and its
// x0 frames. With base == nullptr only the size of both sets is computed.
struct HostSet {
  float* noise;                      // [S][4][4][H][W]
  float* motion;                     // [S][4][512]
  void* hidden[PL_MAX_LAYERS];       // fp16 [S][16][N_l][C_l]
  float* eps;                        // [S][16][4][H][W]
  float* out;                        // [S][4][4][H][W]
  size_t hidden_bytes[PL_MAX_LAYERS];
};

size_t host_layout(const pl_config& c, uint8_t* base, int set, HostSet* hs) {
  const int64_t S = c.sessions > 0 ? c.sessions : 1;
  const int64_t fe = static_cast<int64_t>(c.latent_c) * c.latent_h * c.latent_w;
  size_t off = 0;
  auto take = [&](size_t bytes) -> uint8_t* {
    uint8_t* q = base ? base + off : nullptr;
    off += align_up(bytes);
    return q;
  };
  HostSet h{};
  for (int b = 0; b <= set; ++b) {
    h.noise = reinterpret_cast<float*>(take(sizeof(float) * S * 4 * fe));
    h.motion = reinterpret_cast<float*>(take(sizeof(float) * S * 4 * 512));
    for (int l = 0; l < c.n_layers; ++l) {
      h.hidden_bytes[l] = sizeof(__half) * S * 16 * c.layer_tokens[l] * c.layer_channels[l];
      h.hidden[l] = take(h.hidden_bytes[l]);
    }
    h.eps = reinterpret_cast<float*>(take(sizeof(float) * S * 16 * fe));
    h.out = reinterpret_cast<float*>(take(sizeof(float) * S * 4 * fe));
  }
  if (hs) *hs = h;
  return off;
}

}  // namespace

extern "C" {

const char* pl_status_string(int status) {
  switch (status) {
    case PL_OK: return "ok";
    case PL_EINVAL: return "invalid argument";
    case PL_ESTATE: return "invalid state (call order)";
    case PL_ENOMEM: return "workspace too small";
    case PL_ECUDA: return "CUDA error";
    case PL_ETIMEOUT: return "device wait timed out";
    case PL_EDEVICE: return "device-side contract violation";
    case PL_EUNSUPPORTED: return "unsupported shape";
    default: return "unknown status";
  }
}

int pl_abi_version(void) { return 3; }

pl_status pl_gemm_f16(const void* a, int64_t lda, const void* b, int64_t ldb, void* c,
                      int64_t ldc, int M, int N, int K, void* stream) {
  if (!a || !b || !c) return PL_EINVAL;
  return single_gemm(a, lda, b, ldb, c, ldc, M, N, K, pl::call_status_word(),
                     static_cast<cudaStream_t>(stream));
}

pl_status pl_segment_attention(const void* q, int64_t ldq, int64_t q_frame_stride,
                               const pl_kv_segment* segs, int n_segs, int frames, int n_q,
                               int heads, int head_dim, void* out, int64_t ldo,
                               int64_t out_frame_stride, void* stream) {
  if (!q || !segs || !out) return PL_EINVAL;
  if (n_segs < 1 || n_segs > pl::kAttnMaxSegs) return PL_EINVAL;
  if (!head_dim_supported(head_dim)) return PL_EUNSUPPORTED;
  if (frames > 65535 || heads > 65535) return PL_EINVAL;
  AttnSegHost hs[pl::kAttnMaxSegs];
  for (int i = 0; i < n_segs; ++i) {
    if (!segs[i].k || !segs[i].v) return PL_EINVAL;
    hs[i] = {segs[i].k, segs[i].v, segs[i].len, segs[i].ld, segs[i].frame_stride};
  }
  AttnParams p;
  const int r = pl::attn_make_params(&p, q, ldq, q_frame_stride, hs, n_segs, frames, n_q, heads,
                                     head_dim, out, ldo, out_frame_stride);
  if (r) return r == 1 ? PL_EINVAL : PL_ECUDA;
  p.status = pl::call_status_word();
  const int lr = pl::attn_launch(p, head_dim, static_cast<cudaStream_t>(stream));
  return lr == 0 ? PL_OK : lr == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
}

pl_status pl_test_segment_attention_fault(const void* q, int64_t ldq, int64_t q_frame_stride,
                                         const pl_kv_segment* segs, int n_segs, int frames,
                                         int n_q, int heads, int head_dim, void* out,
                                         int64_t ldo, int64_t out_frame_stride, int mode,
                                         uint32_t wait_us, void* stream) {
  if (!q || !segs || !out) return PL_EINVAL;
  if (mode != PL_TEST_NO_KV && mode != PL_TEST_BAD_BOX) return PL_EINVAL;
  if (wait_us < 1 || wait_us > 2000000) return PL_EINVAL;
  if (n_segs < 1 || n_segs > pl::kAttnMaxSegs) return PL_EINVAL;
  if (!head_dim_supported(head_dim)) return PL_EUNSUPPORTED;
  if (frames > 65535 || heads > 65535) return PL_EINVAL;
  AttnSegHost hs[pl::kAttnMaxSegs];
  for (int i = 0; i < n_segs; ++i) {
    if (!segs[i].k || !segs[i].v) return PL_EINVAL;
    hs[i] = {segs[i].k, segs[i].v, segs[i].len, segs[i].ld, segs[i].frame_stride};
  }
  AttnParams p;
  const int r = pl::attn_make_params(&p, q, ldq, q_frame_stride, hs, n_segs, frames, n_q, heads,
                                     head_dim, out, ldo, out_frame_stride);
  if (r) return r == 1 ? PL_EINVAL : PL_ECUDA;
  p.status = pl::call_status_word();
  p.wait_ns = static_cast<uint64_t>(wait_us) * 1000ull;
  if (mode == PL_TEST_NO_KV) {
    p.test_mode = pl::kTestNoKV;
  } else {
    // the tensor maps stay as encoded; only the count the kernel checks
    // against its key tile is off, so it returns before any copy
    p.box_rows += 16;
  }
  const int lr = pl::attn_launch(p, head_dim, static_cast<cudaStream_t>(stream));
  return lr == 0 ? PL_OK : lr == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
}

pl_status pl_pr_sink_attention(const void* q, const void* k_own, const void* v_own,
                               const void* k_sink, const void* v_sink, const void* k_pool,
                               const void* v_pool, int n_pool, const float* pose_store,
                               const float* pose_query, int pose_dim,
                               const void* const* k_roll, const void* const* v_roll,
                               int n_roll, int n, int heads, int head_dim, void* out,
                               int32_t* retrieved, double* retrieved_d2, void* stream) {
  if (!q || !k_own || !v_own || !k_sink || !v_sink || !k_pool || !v_pool || !pose_store ||
      !pose_query || !out || !retrieved)
    return PL_EINVAL;
  if (n_pool < 1 || n_pool > 65536 || pose_dim < 1 || pose_dim > 4096 || n < 1 || heads < 1)
    return PL_EINVAL;
  if (n_roll < 0 || n_roll > pl::kAttnMaxSegs - 3 || (n_roll > 0 && (!k_roll || !v_roll)))
    return PL_EINVAL;
  if (!head_dim_supported(head_dim)) return PL_EUNSUPPORTED;
  const int64_t ld = static_cast<int64_t>(heads) * head_dim;
  AttnSegHost segs[pl::kAttnMaxSegs];
  int ns = 0;
  segs[ns++] = {k_own, v_own, n, ld, 0};
  segs[ns++] = {k_sink, v_sink, n, ld, 0};
  AttnSegHost pool{k_pool, v_pool, n, ld, static_cast<int64_t>(n) * ld};
  pool.n_blocks = n_pool;
  pool.block_sel = retrieved;
  segs[ns++] = pool;
  for (int r = 0; r < n_roll; ++r) {
    if (!k_roll[r] || !v_roll[r]) return PL_EINVAL;
    segs[ns++] = {k_roll[r], v_roll[r], n, ld, 0};
  }
  AttnParams p;
  const int mr = pl::attn_make_params(&p, q, ld, static_cast<int64_t>(n) * ld, segs, ns, 1, n,
                                      heads, head_dim, out, ld, static_cast<int64_t>(n) * ld);
  if (mr) return mr == 1 ? PL_EINVAL : PL_ECUDA;
  p.status = pl::call_status_word();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pl_status r = from_cuda(pl::launch_nearest(pose_store, n_pool, pose_dim, pose_query, retrieved,
                                             retrieved_d2, s));
  if (r) return r;
  const int lr = pl::attn_launch(p, head_dim, s);
  return lr == 0 ? PL_OK : lr == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
}

pl_status pl_ref_attention_workspace_bytes(int frames, int n, int c, int n_bank, size_t* bytes) {
  if (!bytes || frames < 1 || n < 1 || c < 1 || n_bank < 0 || n_bank > PL_MAX_BANK)
    return PL_EINVAL;
  const size_t fnc = static_cast<size_t>(frames) * n * c;
  *bytes = align_up(2 * 3 * fnc) + align_up(2 * static_cast<size_t>(n_bank) * n * 2 * c) +
           align_up(2 * fnc);
  return PL_OK;
}

pl_status pl_ref_attention(const void* hidden, const void* w_qkv, const void* w_o,
                           const void* const* bank_feats, int n_bank, int frames, int n, int c,
                           int heads, void* out, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!hidden || !w_qkv || !w_o || !out || !workspace) return PL_EINVAL;
  if (heads < 1 || c % heads || c % 16) return PL_EINVAL;
  if (n_bank < 0 || n_bank > PL_MAX_BANK || (n_bank > 0 && !bank_feats)) return PL_EINVAL;
  const int hd = c / heads;
  if (!head_dim_supported(hd)) return PL_EUNSUPPORTED;
  size_t need = 0;
  if (pl_ref_attention_workspace_bytes(frames, n, c, n_bank, &need)) return PL_EINVAL;
  if (workspace_bytes < need) return PL_ENOMEM;
  if (!aligned16(workspace)) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t fnc = static_cast<size_t>(frames) * n * c;
  __half* qkv = static_cast<__half*>(workspace);
  __half* bkv = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(workspace) +
                                          align_up(2 * 3 * fnc));
  __half* o = reinterpret_cast<__half*>(reinterpret_cast<uint8_t*>(bkv) +
                                        align_up(2 * static_cast<size_t>(n_bank) * n * 2 * c));
  uint32_t* status = pl::call_status_word();
  GemmParams gp;
  std::memset(&gp, 0, sizeof(gp));
  gp.status = status;
  int r = pl::gemm_make_problem(&gp.prob[0], hidden, c, w_qkv, 3 * c, qkv, 3 * c, frames * n,
                                3 * c, c, nullptr);
  if (r) return gemm_status(r);
  for (int b = 0; b < n_bank; ++b) {
    if (!bank_feats[b]) return PL_EINVAL;
    r = pl::gemm_make_problem(&gp.prob[1 + b], bank_feats[b], c,
                              static_cast<const __half*>(w_qkv) + c, 3 * c,
                              bkv + static_cast<int64_t>(b) * n * 2 * c, 2 * c, n, 2 * c, c,
                              nullptr);
    if (r) return gemm_status(r);
  }
  gp.n_problems = 1 + n_bank;
  r = pl::gemm_launch(&gp, s, num_sms());
  if (r) return gemm_status(r);
  AttnSegHost segs[1 + PL_MAX_BANK];
  segs[0] = {qkv + c, qkv + 2 * c, n, 3ll * c, static_cast<int64_t>(n) * 3 * c};
  for (int b = 0; b < n_bank; ++b) {
    const __half* kv = bkv + static_cast<int64_t>(b) * n * 2 * c;
    segs[1 + b] = {kv, kv + c, n, 2ll * c, 0};
  }
  AttnParams ap;
  r = pl::attn_make_params(&ap, qkv, 3ll * c, static_cast<int64_t>(n) * 3 * c, segs, 1 + n_bank,
                           frames, n, heads, hd, o, c, static_cast<int64_t>(n) * c);
  if (r) return r == 1 ? PL_EINVAL : PL_ECUDA;
  ap.status = status;
  r = pl::attn_launch(ap, hd, s);
  if (r) return r == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
  return single_gemm(o, c, w_o, c, out, c, frames * n, c, c, status, s);
}

pl_status pl_motion_xattn_workspace_bytes(int frames, int n, int c, size_t* bytes) {
  if (!bytes || frames < 1 || n < 1 || c < 1) return PL_EINVAL;
  const size_t fnc = static_cast<size_t>(frames) * n * c;
  *bytes = align_up(4 * static_cast<size_t>(frames) * 32 * 2 * c) + align_up(4 * fnc) +
           align_up(2 * fnc);
  return PL_OK;
}

pl_status pl_motion_xattn(const void* x, const float* motion, const void* m_q, const void* m_kv,
                          const void* m_o, int frames, int n, int c, int heads, void* out,
                          void* workspace, size_t workspace_bytes, void* stream) {
  if (!x || !motion || !m_q || !m_kv || !m_o || !out || !workspace) return PL_EINVAL;
  if (heads < 1 || c % heads || c % 16 || frames < 1 || frames > 65535 || n < 1) return PL_EINVAL;
  if (!head_dim_supported(c / heads)) return PL_EUNSUPPORTED;
  size_t need = 0;
  if (pl_motion_xattn_workspace_bytes(frames, n, c, &need)) return PL_EINVAL;
  if (workspace_bytes < need) return PL_ENOMEM;
  if (!aligned16(workspace)) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t fnc = static_cast<size_t>(frames) * n * c;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  float* kv = reinterpret_cast<float*>(w);
  w += align_up(4 * static_cast<size_t>(frames) * 32 * 2 * c);
  float* qm = reinterpret_cast<float*>(w);
  w += align_up(4 * fnc);
  __half* om = reinterpret_cast<__half*>(w);
  uint32_t* status = pl::call_status_word();
  pl_status r = from_cuda(pl::launch_motion_kv(motion, static_cast<const __half*>(m_kv), frames,
                                               c, kv, s));
  if (r) return r;
  r = single_gemm(x, c, m_q, c, qm, c, frames * n, c, c, status, s, /*out_f32=*/true);
  if (r) return r;
  r = from_cuda(pl::launch_motion_attn(qm, c, kv, frames, n, c, heads, om, c, s));
  if (r) return r;
  return single_gemm(om, c, m_o, c, out, c, frames * n, c, c, status, s);
}

pl_status pl_motion_bank_check_workspace_bytes(int capacity, int dim, int n_queries,
                                               size_t* bytes) {
  if (!bytes || capacity < 1 || capacity > (1 << 24) || dim < 1 || dim > 4096) return PL_EINVAL;
  if (n_queries < 0 || n_queries > 64) return PL_EINVAL;
  *bytes = n_queries == 0 ? 0 : pl::bank_workspace_bytes(capacity, n_queries);
  return PL_OK;
}

pl_status pl_motion_bank_check(float* bank, int32_t* count, int32_t* appends, int capacity,
                               int dim, const float* queries, int n_queries, float threshold,
                               int cap, int32_t* argmin, double* min_d2, uint8_t* appended,
                               void* workspace, size_t workspace_bytes, void* stream) {
  if (!bank || !count || !appends || (n_queries > 0 && !queries)) return PL_EINVAL;
  if (dim < 1 || dim > 4096 || capacity < 1 || capacity > (1 << 24)) return PL_EINVAL;
  if (n_queries < 0 || n_queries > 64 || cap < 0) return PL_EINVAL;
  if (!(threshold >= 0.f) || !std::isfinite(threshold)) return PL_EINVAL;
  if (n_queries == 0) return PL_OK;
  size_t need = 0;
  if (pl_motion_bank_check_workspace_bytes(capacity, dim, n_queries, &need)) return PL_EINVAL;
  if (need > 0) {
    if (!workspace || !aligned16(workspace)) return PL_EINVAL;
    if (workspace_bytes < need) return PL_ENOMEM;
    if (static_cast<size_t>(n_queries) * dim * sizeof(double) > 160 * 1024) return PL_EUNSUPPORTED;
  }
  const double thr2 = static_cast<double>(threshold) * threshold;
  return from_cuda(pl::launch_bank_check(bank, count, appends, capacity, dim, queries, n_queries,
                                         thr2, cap, argmin, min_d2, appended, nullptr, 1,
                                         need > 0 ? workspace : nullptr,
                                         static_cast<cudaStream_t>(stream)));
}

pl_status pl_nearest_workspace_bytes(int64_t count, size_t* bytes) {
  if (!bytes || count < 1 || count >= (1ll << 40)) return PL_EINVAL;
  const int parts = pl::nearest_parts(count);
  *bytes = align_up(sizeof(double) * parts) + align_up(sizeof(int64_t) * parts);
  return PL_OK;
}

pl_status pl_nearest(const float* store, int64_t count, int dim, const float* query,
                     int64_t* argmin, double* min_d2, void* workspace, size_t workspace_bytes,
                     void* stream) {
  if (!store || !query || !argmin || !workspace) return PL_EINVAL;
  if (dim < 1 || dim > 65536) return PL_EINVAL;
  size_t need = 0;
  const pl_status v = pl_nearest_workspace_bytes(count, &need);
  if (v) return v;
  if (workspace_bytes < need) return PL_ENOMEM;
  if (dim % 4 == 0 && (!aligned16(store) || !aligned16(query))) return PL_EINVAL;
  const int parts = pl::nearest_parts(count);
  double* pd = static_cast<double*>(workspace);
  int64_t* pi = reinterpret_cast<int64_t*>(static_cast<uint8_t*>(workspace) +
                                           align_up(sizeof(double) * parts));
  return from_cuda(pl::launch_nearest_large(store, count, dim, query, pd, pi, parts, argmin,
                                            min_d2, static_cast<cudaStream_t>(stream)));
}

pl_status pl_workspace_bytes(const pl_config* cfg, size_t* bytes) {
  if (!bytes) return PL_EINVAL;
  const pl_status v = validate_config(cfg);
  if (v) return v;
  *bytes = layout(*cfg, nullptr);
  return PL_OK;
}

pl_status pl_ctx_create(const pl_config* cfg, void* workspace, size_t workspace_bytes,
                        pl_ctx** out) {
  if (!out || !workspace) return PL_EINVAL;
  *out = nullptr;
  const pl_status v = validate_config(cfg);
  if (v) return v;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return PL_EINVAL;
  const size_t need = layout(*cfg, nullptr);
  if (workspace_bytes < need) return PL_ENOMEM;
  pl_ctx* ctx = new (std::nothrow) pl_ctx;
  if (!ctx) return PL_ENOMEM;
  std::memset(static_cast<void*>(ctx), 0, sizeof(*ctx));
  ctx->cfg = *cfg;
  ctx->sessions = cfg->sessions > 0 ? cfg->sessions : 1;
  ctx->capacity = 1 + cfg->append_cap;
  ctx->motion_blocks = cfg->motion_blocks == 2 ? 2 : 1;
  ctx->last_round_kernels = -1;
  ctx->frame_elems = static_cast<int64_t>(cfg->latent_c) * cfg->latent_h * cfg->latent_w;
  ctx->ws = static_cast<uint8_t*>(workspace);
  ctx->ws_bytes = workspace_bytes;
  layout(*cfg, ctx);
  pl::ddim_coefficients(&ctx->coef);
  // kernel attributes, the SM count and the call status word are set up here,
  // outside any stream capture
  num_sms();
  pl::call_status_word();
  if (pl::gemm_init() || pl::attn_init()) {
    delete ctx;
    return PL_ECUDA;
  }
  // the round's other streams and their fork / join events
  bool made = cudaEventCreateWithFlags(&ctx->ev_fork, cudaEventDisableTiming) == cudaSuccess;
  for (int k = 0; made && k + 1 < kRoundStreams; ++k)
    made = cudaStreamCreateWithFlags(&ctx->side[k], cudaStreamNonBlocking) == cudaSuccess &&
           cudaEventCreateWithFlags(&ctx->ev_join[k], cudaEventDisableTiming) == cudaSuccess;
  if (!made) {
    pl_ctx_destroy(ctx);
    return PL_ECUDA;
  }
  {
    const char* prof = std::getenv("PL_PROFILE");
    ctx->profile = prof && prof[0] == '1';
  }
  // zero the device state so pl_get_state is meaningful before bank_init
  if (cudaMemset(ctx->st, 0, sizeof(pl::DevState) * ctx->sessions) != cudaSuccess) {
    delete ctx;
    return PL_ECUDA;
  }
  *out = ctx;
  return PL_OK;
}

pl_status pl_ctx_destroy(pl_ctx* ctx) {
  if (!ctx) return PL_OK;
  drop_graph(ctx);
  // the staging the copies write belongs to the caller: finish them first
  if (ctx->copy_stream) cudaStreamSynchronize(ctx->copy_stream);
  for (int b = 0; b < 2; ++b) {
    if (ctx->ev_in[b]) cudaEventDestroy(ctx->ev_in[b]);
    if (ctx->ev_free[b]) cudaEventDestroy(ctx->ev_free[b]);
  }
  if (ctx->copy_stream) cudaStreamDestroy(ctx->copy_stream);
  for (int k = 0; k + 1 < kRoundStreams; ++k) {
    if (ctx->side[k]) {
      cudaStreamSynchronize(ctx->side[k]);
      cudaStreamDestroy(ctx->side[k]);
    }
    if (ctx->ev_join[k]) cudaEventDestroy(ctx->ev_join[k]);
  }
  if (ctx->ev_fork) cudaEventDestroy(ctx->ev_fork);
  for (auto& e : ctx->prof_ev)
    if (e) cudaEventDestroy(e);
  delete ctx;
  return PL_OK;
}

pl_status pl_bank_init(pl_ctx* ctx, const pl_layer_weights* weights,
                       const void* const* ref_feats, const void* const* anchor_feats,
                       const float* ref_motion, const float* drive0_motion,
                       const float* ref_latent, const float* prefill_eps, void* stream) {
  if (!ctx || !ref_motion || !drive0_motion || !ref_latent || !prefill_eps) return PL_EINVAL;
  const int L = ctx->cfg.n_layers;
  if (L > 0 && (!weights || !ref_feats)) return PL_EINVAL;
  for (int l = 0; l < L; ++l) {
    const pl_layer_weights& w = weights[l];
    if (!w.w_qkv || !w.w_o || !w.m_q || !w.m_kv || !w.m_o || !ref_feats[l]) return PL_EINVAL;
    if (ctx->motion_blocks == 2 && (!w.m2_q || !w.m2_kv || !w.m2_o)) return PL_EINVAL;
    ctx->w[l] = w;
    ctx->ref_feats[l] = ref_feats[l];
  }
  ctx->have_anchors = anchor_feats != nullptr && L > 0 && ctx->cfg.append_cap > 0;
  if (ctx->have_anchors) {
    for (int a = 0; a < ctx->cfg.append_cap; ++a)
      for (int l = 0; l < L; ++l) {
        ctx->anchor_feats[a][l] = anchor_feats[a * L + l];
        if (!ctx->anchor_feats[a][l]) return PL_EINVAL;
      }
  }
  drop_graph(ctx);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pl_status r = from_cuda(pl::launch_prefill(ctx->st, ctx->ring, ctx->slot_motion, ctx->bank,
                                             ref_latent, prefill_eps, ref_motion, drive0_motion,
                                             ctx->frame_elems, ctx->capacity, ctx->sessions, s));
  if (r) return r;
  if (L > 0) {
    r = project_bank(ctx, ctx->ref_feats, 0, /*predicated=*/false, s);
    if (r) return r;
  }
  // the folded projections Wo Mq (and Mo Mq2), fp32 accumulation, one rounding
  for (int l = 0; l < L; ++l) {
    const int C = ctx->cfg.layer_channels[l];
    const pl_layer_weights& w = ctx->w[l];
    r = single_gemm(w.w_o, C, w.m_q, C, ctx->w_oq[l], C, C, C, C, &ctx->st->status, s);
    if (r) return r;
    if (ctx->motion_blocks == 2) {
      r = single_gemm(w.m_o, C, w.m2_q, C, ctx->w_oq2[l], C, C, C, C, &ctx->st->status, s);
      if (r) return r;
    }
  }
  ctx->initialised = true;
  return PL_OK;
}

pl_status pl_ring_push(pl_ctx* ctx, const float* new_noise, const float* new_motion,
                       void* stream) {
  if (!ctx || !new_noise || !new_motion) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  return from_cuda(pl::launch_ring_push(ctx->st, ctx->ring, ctx->slot_motion, ctx->batch_motion,
                                        new_noise, new_motion, ctx->frame_elems, ctx->sessions,
                                        static_cast<cudaStream_t>(stream)));
}

pl_status pl_pyramid_ddim_step(pl_ctx* ctx, const float* eps, float* out_x0, void* stream) {
  if (!ctx || !eps || !out_x0) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  if (!aligned16(eps) || !aligned16(out_x0)) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  pl_status r = from_cuda(pl::launch_ddim(ctx->st, ctx->ring, eps, out_x0, ctx->frame_elems,
                                          ctx->coef, ctx->sessions, s));
  if (r) return r;
  return from_cuda(pl::launch_ring_commit(ctx->st, ctx->sessions, s));
}

pl_status pl_ctx_bank_check(pl_ctx* ctx, const float* queries, int n_queries, int32_t* argmin,
                            double* min_d2, uint8_t* appended, void* stream) {
  if (!ctx || (n_queries > 0 && !queries) || n_queries < 0 || n_queries > 64) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  if (n_queries == 0) return PL_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const pl_config& c = ctx->cfg;
  pl_status r = from_cuda(pl::launch_bank_check(
      ctx->bank, nullptr, nullptr, ctx->capacity, 512, queries, n_queries,
      static_cast<double>(c.drift_threshold) * c.drift_threshold, c.append_cap, argmin, min_d2,
      appended, ctx->st, ctx->sessions, nullptr, s));
  if (r) return r;
  if (ctx->have_anchors) {
    for (int an = 1; an <= c.append_cap; ++an) {
      r = project_bank(ctx, ctx->anchor_feats[an - 1], an, /*predicated=*/true, s);
      if (r) return r;
    }
  }
  return PL_OK;
}

pl_status pl_stream_round(pl_ctx* ctx, const float* new_noise, const float* new_motion,
                          const void* const* hidden, const float* eps, float* out_frames,
                          uint8_t* appended, void* const* layer_out, void* const* attn_out,
                          void* stream) {
  if (!ctx || !new_noise || !new_motion || !eps || !out_frames) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  const int L = ctx->cfg.n_layers;
  if (L > 0 && !hidden) return PL_EINVAL;
  for (int l = 0; l < L; ++l) {
    if (!hidden[l] || !aligned16(hidden[l])) return PL_EINVAL;
    if (layer_out && (!layer_out[l] || !aligned16(layer_out[l]))) return PL_EINVAL;
    if (attn_out && (!attn_out[l] || !aligned16(attn_out[l]))) return PL_EINVAL;
  }
  if (!aligned16(new_noise) || !aligned16(eps) || !aligned16(out_frames)) return PL_EINVAL;
  RoundArgs a{new_noise, new_motion, hidden, eps, out_frames, appended, layer_out, attn_out,
              nullptr};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ctx->profile) {
    // profiled rounds run outside the graph, with an event around each layer
    for (int i = 0; i <= L; ++i)
      if (!ctx->prof_ev[i] && cudaEventCreate(&ctx->prof_ev[i]) != cudaSuccess) return PL_ECUDA;
    a.layer_events = ctx->prof_ev;
    ctx->prof_valid = false;
    const pl_status r = enqueue_round(ctx, a, s);
    ctx->prof_valid = r == PL_OK && L > 0;
    return r;
  }
  const char* env = std::getenv("PL_NO_GRAPH");
  const bool use_graph = s != nullptr && !(env && env[0] == '1');
  if (!use_graph) return enqueue_round(ctx, a, s);
  // key = every pointer the captured launches bake in
  static_assert(7 + 3 * PL_MAX_LAYERS <= 64, "graph key size");
  const void* key[64];
  int kn = 0;
  key[kn++] = new_noise;
  key[kn++] = new_motion;
  key[kn++] = eps;
  key[kn++] = out_frames;
  key[kn++] = appended;
  key[kn++] = layer_out ? reinterpret_cast<const void*>(1) : nullptr;
  key[kn++] = attn_out ? reinterpret_cast<const void*>(1) : nullptr;
  for (int l = 0; l < L; ++l) {
    key[kn++] = hidden[l];
    key[kn++] = layer_out ? layer_out[l] : nullptr;
    key[kn++] = attn_out ? attn_out[l] : nullptr;
  }
  pl_ctx::GraphSlot* slot = nullptr;
  for (auto& g : ctx->graphs) {
    bool hit = g.exec && g.key_n == kn;
    for (int i = 0; hit && i < kn; ++i) hit = g.key[i] == key[i];
    if (hit) slot = &g;
  }
  if (!slot) {
    // replace the empty or least recently used capture
    slot = &ctx->graphs[0];
    for (auto& g : ctx->graphs)
      if (!g.exec || (slot->exec && g.last_use < slot->last_use)) slot = &g;
    drop_slot(*slot);
    if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess)
      return PL_ECUDA;
    const pl_status r = enqueue_round(ctx, a, s);
    cudaGraph_t g = nullptr;
    const cudaError_t e = cudaStreamEndCapture(s, &g);
    if (r != PL_OK) {
      if (g) cudaGraphDestroy(g);
      return r;
    }
    if (e != cudaSuccess || !g) return PL_ECUDA;
    if (cudaGraphInstantiate(&slot->exec, g, 0) != cudaSuccess) {
      cudaGraphDestroy(g);
      slot->exec = nullptr;
      return PL_ECUDA;
    }
    slot->graph = g;
    slot->kernels = count_kernel_nodes(g);
    std::memcpy(slot->key, key, sizeof(const void*) * kn);
    slot->key_n = kn;
  }
  slot->last_use = ++ctx->graph_tick;
  ctx->last_round_kernels = slot->kernels;
  return from_cuda(cudaGraphLaunch(slot->exec, s));
}

// ---------------------------------------------------------------- snapshots
namespace {

constexpr uint64_t kSnapMagic = 0x3130504e53504c50ull;   // "PLSNP01" + version byte
constexpr uint32_t kSnapVersion = 1;

struct SnapHeader {
  uint64_t magic;
  uint32_t version, sessions;
  int32_t capacity, latent_c, latent_h, latent_w;
  uint64_t state_bytes, ring_bytes, motion_bytes, bank_bytes;
};

struct SnapParts {
  size_t state, ring, motion, bank, total;
};

SnapParts snap_parts(const pl_ctx* ctx) {
  SnapParts p;
  const size_t S = static_cast<size_t>(ctx->sessions);
  p.state = sizeof(pl::DevState) * S;
  p.ring = sizeof(float) * S * 16 * static_cast<size_t>(ctx->frame_elems);
  p.motion = sizeof(float) * S * 16 * 512;
  p.bank = sizeof(float) * S * static_cast<size_t>(ctx->capacity) * 512;
  p.total = sizeof(SnapHeader) + p.state + p.ring + p.motion + p.bank;
  return p;
}

}  // namespace

pl_status pl_state_bytes(const pl_ctx* ctx, size_t* bytes) {
  if (!ctx || !bytes) return PL_EINVAL;
  *bytes = snap_parts(ctx).total;
  return PL_OK;
}

pl_status pl_state_export(pl_ctx* ctx, void* host_out, size_t bytes, void* stream) {
  if (!ctx || !host_out) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  const SnapParts sp = snap_parts(ctx);
  if (bytes < sp.total) return PL_ENOMEM;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PL_ECUDA;
  SnapHeader h{};
  h.magic = kSnapMagic;
  h.version = kSnapVersion;
  h.sessions = static_cast<uint32_t>(ctx->sessions);
  h.capacity = ctx->capacity;
  h.latent_c = ctx->cfg.latent_c;
  h.latent_h = ctx->cfg.latent_h;
  h.latent_w = ctx->cfg.latent_w;
  h.state_bytes = sp.state;
  h.ring_bytes = sp.ring;
  h.motion_bytes = sp.motion;
  h.bank_bytes = sp.bank;
  uint8_t* o = static_cast<uint8_t*>(host_out);
  std::memcpy(o, &h, sizeof(h));
  o += sizeof(h);
  const struct {
    const void* src;
    size_t n;
  } parts[4] = {{ctx->st, sp.state}, {ctx->ring, sp.ring}, {ctx->slot_motion, sp.motion},
                {ctx->bank, sp.bank}};
  for (const auto& pt : parts) {
    if (cudaMemcpy(o, pt.src, pt.n, cudaMemcpyDeviceToHost) != cudaSuccess) return PL_ECUDA;
    o += pt.n;
  }
  return PL_OK;
}

pl_status pl_state_import(pl_ctx* ctx, const void* host_in, size_t bytes, void* stream) {
  if (!ctx || !host_in) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  const SnapParts sp = snap_parts(ctx);
  if (bytes < sp.total) return PL_EINVAL;
  SnapHeader h;
  std::memcpy(&h, host_in, sizeof(h));
  if (h.magic != kSnapMagic || h.version != kSnapVersion ||
      h.sessions != static_cast<uint32_t>(ctx->sessions) || h.capacity != ctx->capacity ||
      h.latent_c != ctx->cfg.latent_c || h.latent_h != ctx->cfg.latent_h ||
      h.latent_w != ctx->cfg.latent_w || h.state_bytes != sp.state || h.ring_bytes != sp.ring ||
      h.motion_bytes != sp.motion || h.bank_bytes != sp.bank)
    return PL_EINVAL;
  const uint8_t* in = static_cast<const uint8_t*>(host_in) + sizeof(h);
  // the states are checked on the host before anything reaches the device
  const int S = ctx->sessions;
  pl::DevState* states = new (std::nothrow) pl::DevState[S];
  if (!states) return PL_ENOMEM;
  std::memcpy(states, in, sp.state);
  for (int z = 0; z < S; ++z) {
    pl::DevState& d = states[z];
    bool ok = d.head >= 0 && d.head < 4 && d.bank_count >= 1 && d.bank_count <= ctx->capacity &&
              d.appends >= 0 && d.appends <= ctx->cfg.append_cap &&
              d.bank_count == 1 + d.appends && d.rounds >= 0;
    for (int i = 0; i < 4; ++i) {
      const int t = d.slot_t[i];
      ok = ok && (t == -1 || t == 0 || t == 333 || t == 666 || t == 999);
    }
    if (!ok) {
      delete[] states;
      return PL_EINVAL;
    }
    d.status = 0;
    for (int a = 0; a < 4; ++a) d.anchor_fire[a] = 0;
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemcpy(ctx->st, states, sp.state, cudaMemcpyHostToDevice);
  in += sp.state;
  if (e == cudaSuccess) e = cudaMemcpy(ctx->ring, in, sp.ring, cudaMemcpyHostToDevice);
  in += sp.ring;
  if (e == cudaSuccess) e = cudaMemcpy(ctx->slot_motion, in, sp.motion, cudaMemcpyHostToDevice);
  in += sp.motion;
  if (e == cudaSuccess) e = cudaMemcpy(ctx->bank, in, sp.bank, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) {
    delete[] states;
    return PL_ECUDA;
  }
  // KV-bank entries 1..appends hold anchors 1..appends projected by each
  // layer's Wk/Wv: recompute them rather than carry ~185 MB in the snapshot
  pl_status r = PL_OK;
  if (ctx->have_anchors) {
    for (int z = 0; z < S && r == PL_OK; ++z)
      for (int an = 1; an <= states[z].appends && r == PL_OK; ++an)
        r = project_bank(ctx, ctx->anchor_feats[an - 1], an, /*predicated=*/false, s, z);
  }
  delete[] states;
  return r;
}

pl_status pl_host_staging_bytes(const pl_config* cfg, size_t* bytes) {
  if (!bytes) return PL_EINVAL;
  const pl_status v = validate_config(cfg);
  if (v) return v;
  *bytes = host_layout(*cfg, nullptr, 1, nullptr);
  return PL_OK;
}

pl_status pl_stream_round_host(pl_ctx* ctx, void* staging, size_t staging_bytes,
                               const float* h_noise, const float* h_motion,
                               const void* const* h_hidden, const float* h_eps,
                               float* h_out_frames, void* stream) {
  if (!ctx || !staging || !h_noise || !h_motion || !h_eps || !h_out_frames) return PL_EINVAL;
  if (!ctx->initialised) return PL_ESTATE;
  const pl_config& c = ctx->cfg;
  const int L = c.n_layers;
  if (L > 0 && !h_hidden) return PL_EINVAL;
  for (int l = 0; l < L; ++l)
    if (!h_hidden[l]) return PL_EINVAL;
  if (reinterpret_cast<uintptr_t>(staging) % kAlign) return PL_EINVAL;
  if (staging_bytes < host_layout(c, nullptr, 1, nullptr)) return PL_ENOMEM;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!ctx->copy_stream) {
    if (cudaStreamCreateWithFlags(&ctx->copy_stream, cudaStreamNonBlocking) != cudaSuccess)
      return PL_ECUDA;
    for (int b = 0; b < 2; ++b) {
      if (cudaEventCreateWithFlags(&ctx->ev_in[b], cudaEventDisableTiming) != cudaSuccess ||
          cudaEventCreateWithFlags(&ctx->ev_free[b], cudaEventDisableTiming) != cudaSuccess)
        return PL_ECUDA;
    }
  }
  const int b = static_cast<int>(ctx->host_rounds & 1);
  HostSet h;
  host_layout(c, static_cast<uint8_t*>(staging), b, &h);
  const int64_t S = ctx->sessions;
  const size_t fe = static_cast<size_t>(ctx->frame_elems);
  cudaStream_t cs = ctx->copy_stream;
  // set b is refilled once the round that last read it (two calls ago) is done
  if (ctx->free_pending[b] && cudaStreamWaitEvent(cs, ctx->ev_free[b], 0) != cudaSuccess)
    return PL_ECUDA;
  cudaError_t e = cudaMemcpyAsync(h.noise, h_noise, sizeof(float) * S * 4 * fe,
                                  cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h.motion, h_motion, sizeof(float) * S * 4 * 512, cudaMemcpyHostToDevice, cs);
  for (int l = 0; l < L && e == cudaSuccess; ++l)
    e = cudaMemcpyAsync(h.hidden[l], h_hidden[l], h.hidden_bytes[l], cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(h.eps, h_eps, sizeof(float) * S * 16 * fe, cudaMemcpyHostToDevice, cs);
  if (e == cudaSuccess) e = cudaEventRecord(ctx->ev_in[b], cs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ctx->ev_in[b], 0);
  if (e != cudaSuccess) return PL_ECUDA;
  const pl_status r = pl_stream_round(ctx, h.noise, h.motion, h.hidden, h.eps, h.out, nullptr,
                                      nullptr, nullptr, stream);
  if (r != PL_OK) return r;
  if (cudaEventRecord(ctx->ev_free[b], s) != cudaSuccess) return PL_ECUDA;
  ctx->free_pending[b] = true;
  ++ctx->host_rounds;
  return from_cuda(cudaMemcpyAsync(h_out_frames, h.out, sizeof(float) * S * 4 * fe,
                                   cudaMemcpyDeviceToHost, s));
}

pl_status pl_get_session_state(pl_ctx* ctx, int session, pl_state* out, void* stream) {
  if (!ctx || !out || session < 0 || session >= ctx->sessions) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return PL_ECUDA;
  pl::DevState d;
  if (cudaMemcpy(&d, ctx->st + session, sizeof(d), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PL_ECUDA;
  std::memset(out, 0, sizeof(*out));
  out->initialised = ctx->initialised ? d.initialised : 0;
  out->head = d.head;
  for (int i = 0; i < 4; ++i) out->slot_t[i] = d.slot_t[i];
  out->rounds = d.rounds;
  out->frames_in = d.frames_in;
  out->frames_out = d.frames_out;
  out->bank_count = d.bank_count;
  out->appends = d.appends;
  out->device_status = d.status;
  return PL_OK;
}

pl_status pl_get_state(pl_ctx* ctx, pl_state* out, void* stream) {
  return pl_get_session_state(ctx, 0, out, stream);
}

pl_status pl_get_session_motion_bank(pl_ctx* ctx, int session, float* host_out, int32_t* count,
                                     void* stream) {
  if (!ctx || !host_out || !count || session < 0 || session >= ctx->sessions) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return PL_ECUDA;
  int32_t n = 0;
  if (cudaMemcpy(&n, &ctx->st[session].bank_count, sizeof(n), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return PL_ECUDA;
  if (n < 0 || n > ctx->capacity) return PL_EDEVICE;
  *count = n;
  const float* bank = ctx->bank + static_cast<int64_t>(session) * ctx->capacity * 512;
  if (n > 0 &&
      cudaMemcpy(host_out, bank, sizeof(float) * 512 * n, cudaMemcpyDeviceToHost) != cudaSuccess)
    return PL_ECUDA;
  return PL_OK;
}

pl_status pl_get_motion_bank(pl_ctx* ctx, float* host_out, int32_t* count, void* stream) {
  return pl_get_session_motion_bank(ctx, 0, host_out, count, stream);
}

pl_status pl_get_device_status(pl_ctx* ctx, void* stream) {
  if (!ctx) return PL_EINVAL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return PL_ECUDA;
  uint32_t w = 0;
  for (int z = 0; z < ctx->sessions; ++z) {
    uint32_t wz = 0;
    if (cudaMemcpy(&wz, &ctx->st[z].status, sizeof(wz), cudaMemcpyDeviceToHost) != cudaSuccess)
      return PL_ECUDA;
    const uint32_t zero = 0;
    if (cudaMemcpy(&ctx->st[z].status, &zero, sizeof(zero), cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return PL_ECUDA;
    w |= wz;
  }
  if (w & pl::DEV_TIMEOUT) return PL_ETIMEOUT;
  if (w) return PL_EDEVICE;
  return PL_OK;
}

pl_status pl_set_profiling(pl_ctx* ctx, int on) {
  if (!ctx) return PL_EINVAL;
  ctx->profile = on != 0;
  ctx->prof_valid = false;
  return PL_OK;
}

pl_status pl_round_kernel_count(const pl_ctx* ctx, int* count) {
  if (!ctx || !count) return PL_EINVAL;
  if (ctx->last_round_kernels < 0) return PL_ESTATE;
  *count = ctx->last_round_kernels;
  return PL_OK;
}

pl_status pl_get_layer_ms(pl_ctx* ctx, float* ms_out, int n) {
  if (!ctx || !ms_out || n < ctx->cfg.n_layers) return PL_EINVAL;
  if (!ctx->prof_valid) return PL_ESTATE;
  const int L = ctx->cfg.n_layers;
  if (cudaEventSynchronize(ctx->prof_ev[L]) != cudaSuccess) return PL_ECUDA;
  for (int l = 0; l < L; ++l)
    if (cudaEventElapsedTime(&ms_out[l], ctx->prof_ev[l], ctx->prof_ev[l + 1]) != cudaSuccess)
      return PL_ECUDA;
  return PL_OK;
}

pl_status pl_get_call_status(void* stream) {
  uint32_t* word = pl::call_status_word();
  if (!word) return PL_ECUDA;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PL_ECUDA;
  uint32_t w = 0;
  if (cudaMemcpy(&w, word, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess) return PL_ECUDA;
  const uint32_t zero = 0;
  if (cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return PL_ECUDA;
  if (w & pl::DEV_TIMEOUT) return PL_ETIMEOUT;
  if (w) return PL_EDEVICE;
  return PL_OK;
}

const float* pl_ctx_ring_latents(const pl_ctx* ctx) { return ctx ? ctx->ring : nullptr; }

}  // extern "C"
