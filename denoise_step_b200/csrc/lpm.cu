// Pre-rotary KV cache with a sliding window (LPM 1.0 real-time digital actor
// write-up, sections 7.3 "滑动窗口注意力" and 7.4 "Pre-RoPE KV Cache"): the
// context of a new chunk is the reference tokens, three fixed sink chunks
// and the two most recent chunks; K/V are cached before the rotary code and
// K is rotated by each token's position in the current window.
//
// The rotation is one HBM-bound pass per key per step into a rotated-K
// window buffer, not a pass inside the attention: every CTA of a head reads
// the same K tiles, so rotating in the attention's shared memory repeats the
// work once per query tile (measured on B200: 9.7-11.6 ms against 1.97 ms for
// the same attention, whereas the pass costs ~1-4 %). Only what moved is
// rotated again: the reference and the sinks keep their positions, so their
// rotated rows are written once; each step rotates the sliding chunks (their
// positions shift as they age) and the new chunk. V is never rotated and is
// read from the cache in place.
#include <cuda_runtime.h>

#include <cmath>
#include <cstring>
#include <new>

#include "../../include/pl.h"
#include "attn.cuh"
#include "devinit.cuh"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kSinks = 3;     // fixed sink chunks
constexpr int kSlide = 2;     // sliding-window chunks
constexpr int kChunkBlocks = kSinks + kSlide + 1;

bool rope_head_dim(int hd) { return hd == 40 || hd == 64 || hd == 80 || hd == 128 || hd == 160; }

// dst[r] = rotary code of src[r] at position pos0 + r, r < rows: in every
// head the pair (2i, 2i+1) turns by (pos0 + r) * theta_i, (cos, sin) from
// tab[pos][i]. One thread per 4 pairs (16-byte loads and stores; head_dim / 2
// is a multiple of 4 for every supported head_dim); fp32 arithmetic.
__global__ void rope_rows_kernel(const __half* __restrict__ src, int64_t lds,
                                 __half* __restrict__ dst, int64_t ldd, int rows, int heads,
                                 int head_dim, int pos0, const float2* __restrict__ tab) {
  const int half = head_dim / 2;
  const int quads_head = half / 4;
  const int quads_row = heads * quads_head;
  const int64_t total = static_cast<int64_t>(rows) * quads_row;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = k / quads_row;
    const int qr = static_cast<int>(k - r * quads_row);
    const int h = qr / quads_head, i0 = 4 * (qr - h * quads_head);
    const int col = h * head_dim + 2 * i0;
    const float4* t = reinterpret_cast<const float4*>(tab + (pos0 + r) * half + i0);
    const float4 cs01 = __ldg(t), cs23 = __ldg(t + 1);
    const uint4 raw = *reinterpret_cast<const uint4*>(src + r * lds + col);
    const float2 x0 = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
    const float2 x1 = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
    const float2 x2 = __half22float2(*reinterpret_cast<const __half2*>(&raw.z));
    const float2 x3 = __half22float2(*reinterpret_cast<const __half2*>(&raw.w));
    auto turn = [](float2 x, float c, float s) {
      const __half2 y = __floats2half2_rn(x.x * c - x.y * s, x.x * s + x.y * c);
      return *reinterpret_cast<const uint32_t*>(&y);
    };
    uint4 o;
    o.x = turn(x0, cs01.x, cs01.y);
    o.y = turn(x1, cs01.z, cs01.w);
    o.z = turn(x2, cs23.x, cs23.y);
    o.w = turn(x3, cs23.z, cs23.w);
    *reinterpret_cast<uint4*>(dst + r * ldd + col) = o;
  }
}

cudaError_t launch_rope_rows(const __half* src, int64_t lds, __half* dst, int64_t ldd, int rows,
                             int heads, int head_dim, int pos0, const float2* tab,
                             cudaStream_t s) {
  const int64_t total = static_cast<int64_t>(rows) * heads * (head_dim / 8);
  if (total == 0) return cudaSuccess;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  rope_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(src, lds, dst, ldd, rows, heads,
                                                                  head_dim, pos0, tab);
  return cudaGetLastError();
}

// tab[pos][i] = (cos, sin)(pos * base^(-2i / head_dim)), angles in fp64
__global__ void rope_table_kernel(float2* tab, int positions, int half, double log_base,
                                  int head_dim) {
  const int64_t total = static_cast<int64_t>(positions) * half;
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < total;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pos = k / half;
    const int i = static_cast<int>(k - pos * half);
    const double theta = exp(-2.0 * i / head_dim * log_base);
    double sn, cs;
    sincos(static_cast<double>(pos) * theta, &sn, &cs);
    tab[k] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
}

cudaError_t launch_rope_table(float2* tab, int positions, int head_dim, double base,
                              cudaStream_t s) {
  const int half = head_dim / 2;
  const int64_t total = static_cast<int64_t>(positions) * half;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  rope_table_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(tab, positions, half,
                                                                   std::log(base), head_dim);
  return cudaGetLastError();
}

pl_status status_of(int r) {
  return r == 0 ? PL_OK : r == 1 ? PL_EINVAL : r == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
}

struct LpmLayout {
  size_t ref_k, ref_v, k, v, wk, q, tab, total;
};

LpmLayout lpm_layout(int ref_tokens, int chunk_tokens, int heads, int hd) {
  const size_t row = static_cast<size_t>(heads) * hd;
  const int positions = ref_tokens + kChunkBlocks * chunk_tokens;
  LpmLayout l;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
  l.ref_k = take(2 * static_cast<size_t>(ref_tokens) * row);
  l.ref_v = take(2 * static_cast<size_t>(ref_tokens) * row);
  l.k = take(2 * static_cast<size_t>(kChunkBlocks) * chunk_tokens * row);
  l.v = take(2 * static_cast<size_t>(kChunkBlocks) * chunk_tokens * row);
  l.wk = take(2 * static_cast<size_t>(positions) * row);      // rotated K, row = position
  l.q = take(2 * static_cast<size_t>(chunk_tokens) * row);    // rotated queries
  l.tab = take(8 * static_cast<size_t>(positions) * (hd / 2));
  l.total = off;
  return l;
}

pl_status lpm_validate(int ref_tokens, int chunk_tokens, int heads, int hd) {
  if (ref_tokens < 0 || chunk_tokens < 1 || heads < 1 || heads > 65535) return PL_EINVAL;
  if (static_cast<int64_t>(ref_tokens) + static_cast<int64_t>(kChunkBlocks) * chunk_tokens >
      (1ll << 28))
    return PL_EINVAL;
  if (!rope_head_dim(hd)) return PL_EUNSUPPORTED;
  return PL_OK;
}

}  // namespace

struct pl_lpm {
  int ref_tokens, chunk_tokens, heads, hd, positions;
  int64_t chunk_elems;
  __half* ref_k;
  __half* ref_v;
  __half* k;
  __half* v;
  __half* wk;      // rotated K of the window, row = window position
  __half* q_rot;
  float2* tab;
  bool tab_ready;
  bool ref_rotated;
  double base;
  // index lists (host): arena block of each sink, of the sliding chunks (oldest first)
  int sinks[kSinks];
  int n_sink;
  int slide[kSlide];
  int n_slide;
  int reserved;
  bool free_block[kChunkBlocks];
  int64_t chunks;
  int last_q_pos0;
};

extern "C" {

pl_status pl_rope_table(float* tab, int positions, int head_dim, float base, void* stream) {
  if (!tab || positions < 1 || head_dim < 2 || head_dim % 2 || !(base > 1.f) ||
      !std::isfinite(base))
    return PL_EINVAL;
  if (reinterpret_cast<uintptr_t>(tab) & 7) return PL_EINVAL;
  return launch_rope_table(reinterpret_cast<float2*>(tab), positions, head_dim, base,
                           static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? PL_OK
             : PL_ECUDA;
}

pl_status pl_rope_attention_workspace_bytes(int n_q, int64_t total_keys, int heads, int head_dim,
                                            size_t* bytes) {
  if (!bytes || n_q < 1 || total_keys < 1 || heads < 1) return PL_EINVAL;
  const size_t row = static_cast<size_t>(heads) * head_dim;
  *bytes = align_up(2 * static_cast<size_t>(n_q) * row) +
           align_up(2 * static_cast<size_t>(total_keys) * row);
  return PL_OK;
}

pl_status pl_rope_attention(const void* q, int64_t ldq, int q_pos0, const pl_kv_segment* segs,
                            const int64_t* seg_pos0, int n_segs, int n_q, int heads, int head_dim,
                            const float* tab, int tab_positions, void* out, int64_t ldo,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !segs || !seg_pos0 || !tab || !out || !workspace) return PL_EINVAL;
  if (n_segs < 1 || n_segs > pl::kAttnMaxSegs || n_q < 1 || heads < 1 || heads > 65535)
    return PL_EINVAL;
  if (!rope_head_dim(head_dim)) return PL_EUNSUPPORTED;
  if (q_pos0 < 0 || tab_positions < 1 || static_cast<int64_t>(q_pos0) + n_q > tab_positions)
    return PL_EINVAL;
  // 16-byte rows and table entries for the rotation pass
  if (ldq % 8 || ldo % 8 || ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(tab)) & 15))
    return PL_EINVAL;
  int64_t keys = 0;
  for (int s = 0; s < n_segs; ++s) {
    if (!segs[s].k || !segs[s].v || segs[s].frame_stride != 0 || segs[s].len < 1) return PL_EINVAL;
    if (reinterpret_cast<uintptr_t>(segs[s].k) & 15) return PL_EINVAL;
    // the rotated K copy is dense, and the attention reads a segment's K and V
    // with one row stride, so V must be dense too
    if (segs[s].ld != static_cast<int64_t>(heads) * head_dim) return PL_EINVAL;
    if (seg_pos0[s] < 0 || seg_pos0[s] + segs[s].len > tab_positions) return PL_EINVAL;
    keys += segs[s].len;
  }
  size_t need = 0;
  if (pl_rope_attention_workspace_bytes(n_q, keys, heads, head_dim, &need)) return PL_EINVAL;
  if (workspace_bytes < need) return PL_ENOMEM;
  if (reinterpret_cast<uintptr_t>(workspace) % 16) return PL_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t C = static_cast<int64_t>(heads) * head_dim;
  const float2* t2 = reinterpret_cast<const float2*>(tab);
  __half* qr = static_cast<__half*>(workspace);
  __half* kr = reinterpret_cast<__half*>(static_cast<uint8_t*>(workspace) +
                                         align_up(2 * static_cast<size_t>(n_q) * C));
  if (launch_rope_rows(static_cast<const __half*>(q), ldq, qr, C, n_q, heads, head_dim, q_pos0,
                       t2, st) != cudaSuccess)
    return PL_ECUDA;
  pl::AttnSegHost hs[pl::kAttnMaxSegs];
  int64_t off = 0;
  for (int s = 0; s < n_segs; ++s) {
    __half* dst = kr + off * C;
    if (launch_rope_rows(static_cast<const __half*>(segs[s].k), segs[s].ld, dst, C,
                         static_cast<int>(segs[s].len), heads, head_dim,
                         static_cast<int>(seg_pos0[s]), t2, st) != cudaSuccess)
      return PL_ECUDA;
    hs[s] = {dst, segs[s].v, segs[s].len, C, 0};
    off += segs[s].len;
  }
  pl::AttnParams p;
  const int mr = pl::attn_make_params(&p, qr, C, static_cast<int64_t>(n_q) * C, hs, n_segs, 1,
                                      n_q, heads, head_dim, out, ldo,
                                      static_cast<int64_t>(n_q) * ldo);
  if (mr) return mr == 1 ? PL_EINVAL : PL_ECUDA;
  p.status = pl::call_status_word();
  return status_of(pl::attn_launch(p, head_dim, st));
}

pl_status pl_lpm_workspace_bytes(int ref_tokens, int chunk_tokens, int heads, int head_dim,
                                 size_t* bytes) {
  if (!bytes) return PL_EINVAL;
  const pl_status v = lpm_validate(ref_tokens, chunk_tokens, heads, head_dim);
  if (v) return v;
  *bytes = lpm_layout(ref_tokens, chunk_tokens, heads, head_dim).total;
  return PL_OK;
}

pl_status pl_lpm_create(int ref_tokens, int chunk_tokens, int heads, int head_dim,
                        float rope_base, void* workspace, size_t workspace_bytes, pl_lpm** out) {
  if (!out || !workspace) return PL_EINVAL;
  *out = nullptr;
  const pl_status v = lpm_validate(ref_tokens, chunk_tokens, heads, head_dim);
  if (v) return v;
  if (!(rope_base > 1.f) || !std::isfinite(rope_base)) return PL_EINVAL;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return PL_EINVAL;
  const LpmLayout l = lpm_layout(ref_tokens, chunk_tokens, heads, head_dim);
  if (workspace_bytes < l.total) return PL_ENOMEM;
  pl_lpm* m = new (std::nothrow) pl_lpm;
  if (!m) return PL_ENOMEM;
  std::memset(static_cast<void*>(m), 0, sizeof(*m));
  uint8_t* w = static_cast<uint8_t*>(workspace);
  m->ref_tokens = ref_tokens;
  m->chunk_tokens = chunk_tokens;
  m->heads = heads;
  m->hd = head_dim;
  m->positions = ref_tokens + kChunkBlocks * chunk_tokens;
  m->chunk_elems = static_cast<int64_t>(chunk_tokens) * heads * head_dim;
  m->ref_k = reinterpret_cast<__half*>(w + l.ref_k);
  m->ref_v = reinterpret_cast<__half*>(w + l.ref_v);
  m->k = reinterpret_cast<__half*>(w + l.k);
  m->v = reinterpret_cast<__half*>(w + l.v);
  m->wk = reinterpret_cast<__half*>(w + l.wk);
  m->q_rot = reinterpret_cast<__half*>(w + l.q);
  m->tab = reinterpret_cast<float2*>(w + l.tab);
  m->base = rope_base;
  m->tab_ready = false;
  for (int b = 0; b < kChunkBlocks; ++b) m->free_block[b] = true;
  m->reserved = -1;
  m->last_q_pos0 = -1;
  if (pl::attn_init() != 0) {
    delete m;
    return PL_ECUDA;
  }
  *out = m;
  return PL_OK;
}

pl_status pl_lpm_destroy(pl_lpm* m) {
  delete m;
  return PL_OK;
}

pl_status pl_lpm_ref_kv(pl_lpm* m, void** k, void** v) {
  if (!m || !k || !v) return PL_EINVAL;
  if (m->ref_tokens == 0) return PL_EINVAL;
  *k = m->ref_k;
  *v = m->ref_v;
  return PL_OK;
}

pl_status pl_lpm_chunk_kv(pl_lpm* m, void** k, void** v) {
  if (!m || !k || !v) return PL_EINVAL;
  if (m->reserved < 0) {
    for (int b = 0; b < kChunkBlocks; ++b)
      if (m->free_block[b]) {
        m->reserved = b;
        m->free_block[b] = false;
        break;
      }
    if (m->reserved < 0) return PL_ESTATE;   // cannot happen: the arena holds 6 chunks
  }
  *k = m->k + m->reserved * m->chunk_elems;
  *v = m->v + m->reserved * m->chunk_elems;
  return PL_OK;
}

pl_status pl_lpm_step(pl_lpm* m, const void* q, void* out, void* stream) {
  if (!m || !q || !out) return PL_EINVAL;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15) return PL_EINVAL;
  if (m->reserved < 0) return PL_ESTATE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!m->tab_ready) {
    if (launch_rope_table(m->tab, m->positions, m->hd, m->base, st) != cudaSuccess)
      return PL_ECUDA;
    m->tab_ready = true;
  }
  const int64_t C = static_cast<int64_t>(m->heads) * m->hd;
  const int L = m->chunk_tokens;
  // window: [reference ; sinks ; sliding (oldest first) ; current], positions
  // in that order; wk row p holds the rotated K of the token at position p
  pl::AttnSegHost hs[pl::kAttnMaxSegs];
  int ns = 0;
  int pos = 0;
  auto rotate = [&](const __half* src, int rows, int p0) {
    return launch_rope_rows(src, C, m->wk + p0 * C, C, rows, m->heads, m->hd, p0, m->tab, st);
  };
  if (m->ref_tokens > 0) {
    if (!m->ref_rotated) {   // position 0 forever: rotated once
      if (rotate(m->ref_k, m->ref_tokens, 0) != cudaSuccess) return PL_ECUDA;
      m->ref_rotated = true;
    }
    hs[ns++] = {m->wk, m->ref_v, m->ref_tokens, C, 0};
    pos = m->ref_tokens;
  }
  // a sink keeps the position it had as the current chunk: rotated then
  for (int i = 0; i < m->n_sink; ++i, pos += L)
    hs[ns++] = {m->wk + pos * C, m->v + m->sinks[i] * m->chunk_elems, L, C, 0};
  // sliding chunks move each step: rotated again at their new positions
  for (int i = 0; i < m->n_slide; ++i, pos += L) {
    if (rotate(m->k + m->slide[i] * m->chunk_elems, L, pos) != cudaSuccess) return PL_ECUDA;
    hs[ns++] = {m->wk + pos * C, m->v + m->slide[i] * m->chunk_elems, L, C, 0};
  }
  const int q_pos0 = pos;
  if (rotate(m->k + m->reserved * m->chunk_elems, L, pos) != cudaSuccess) return PL_ECUDA;
  hs[ns++] = {m->wk + pos * C, m->v + m->reserved * m->chunk_elems, L, C, 0};
  if (launch_rope_rows(static_cast<const __half*>(q), C, m->q_rot, C, L, m->heads, m->hd, q_pos0,
                       m->tab, st) != cudaSuccess)
    return PL_ECUDA;
  pl::AttnParams p;
  const int mr = pl::attn_make_params(&p, m->q_rot, C, static_cast<int64_t>(L) * C, hs, ns, 1, L,
                                      m->heads, m->hd, out, C, static_cast<int64_t>(L) * C);
  if (mr) return mr == 1 ? PL_EINVAL : PL_ECUDA;
  const pl_status r = status_of(pl::attn_launch(p, m->hd, st));
  if (r) return r;
  // the chunk joins the cache: one of the first three becomes a sink, later
  // ones slide (the oldest of a full window is dropped, its block freed)
  if (m->n_sink < kSinks) {
    m->sinks[m->n_sink++] = m->reserved;
  } else {
    if (m->n_slide == kSlide) {
      m->free_block[m->slide[0]] = true;
      for (int i = 1; i < kSlide; ++i) m->slide[i - 1] = m->slide[i];
      --m->n_slide;
    }
    m->slide[m->n_slide++] = m->reserved;
  }
  m->reserved = -1;
  m->last_q_pos0 = q_pos0;
  ++m->chunks;
  return PL_OK;
}

pl_status pl_lpm_get_state(pl_lpm* m, pl_lpm_state* out) {
  if (!m || !out) return PL_EINVAL;
  std::memset(out, 0, sizeof(*out));
  out->chunks = m->chunks;
  out->n_sink = m->n_sink;
  out->n_slide = m->n_slide;
  out->last_q_pos0 = m->last_q_pos0;
  return PL_OK;
}

}  // extern "C"
