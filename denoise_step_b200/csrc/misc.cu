#include <cmath>

#include "misc.cuh"
#include "ptx.cuh"

namespace pl {

// ------------------------------------------------------------------ schedule
// SD scaled-linear betas (beta_i = (sqrt(0.00085) + i (sqrt(0.012) -
// sqrt(0.00085)) / 999)^2), alpha_bar_t = prod_{i<=t} (1 - beta_i), in fp64.
void ddim_coefficients(DdimCoef* out) {
  double abar[1000];
  const double a = std::sqrt(0.00085), b = std::sqrt(0.012);
  double prod = 1.0;
  for (int i = 0; i < 1000; ++i) {
    const double r = a + i * (b - a) / 999.0;
    prod *= 1.0 - r * r;
    abar[i] = prod;
  }
  const int ts[4] = {999, 666, 333, 0};
  for (int k = 0; k < 4; ++k) {
    const int t = ts[k];
    const double at = abar[t];
    const double ap = t - 333 >= 0 ? abar[t - 333] : 1.0;
    out->c[k][0] = 1.0 / std::sqrt(at);
    out->c[k][1] = std::sqrt(1.0 - at);
    out->c[k][2] = std::sqrt(ap);
    out->c[k][3] = std::sqrt(1.0 - ap);
    out->fwd[k][0] = std::sqrt(at);
    out->fwd[k][1] = std::sqrt(1.0 - at);
  }
}

namespace {

__device__ __forceinline__ int t_index(int t) {  // 999 -> 0, 666 -> 1, 333 -> 2, 0 -> 3
  return t == 999 ? 0 : t == 666 ? 1 : t == 333 ? 2 : t == 0 ? 3 : -1;
}

// ------------------------------------------------------------------ prefill
// 3 windows at t = 0, 333, 666 (oldest first) in slots 0..2; slot 3 free.
// blockIdx.z = session (every buffer carries a leading session dimension).
__global__ void prefill_kernel(DevState* st, float* ring, float* slot_motion, float* bank,
                               const float* __restrict__ ref_latent,
                               const float* __restrict__ prefill_eps,
                               const float* __restrict__ ref_motion,
                               const float* __restrict__ drive0, int64_t frame_elems,
                               int capacity, DdimCoef coef) {
  const int z = blockIdx.z;
  st += z;
  ring += z * 16 * frame_elems;
  slot_motion += z * 16 * 512;
  bank += static_cast<int64_t>(z) * capacity * 512;
  ref_latent += z * frame_elems;
  prefill_eps += z * 12 * frame_elems;
  ref_motion += z * 512;
  drive0 += z * 512;
  const int64_t total = 12 * frame_elems;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t k = i / frame_elems;      // prefill frame 0..11
    const int64_t e = i - k * frame_elems;
    const int w = static_cast<int>(k / 4);  // window 0..2 -> t = 0, 333, 666
    const int ti = 3 - w;                   // table index of t
    const double x = coef.fwd[ti][0] * static_cast<double>(ref_latent[e]) +
                     coef.fwd[ti][1] * static_cast<double>(prefill_eps[i]);
    ring[i] = static_cast<float>(x);        // slot w, frame k % 4
  }
  // motion: 13-point ramp ref -> drive0 with the last point dropped
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 12 * 512;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>(i / 512);
    const int d = static_cast<int>(i % 512);
    const double r = ref_motion[d], t = drive0[d];
    slot_motion[i] = static_cast<float>(r + (static_cast<double>(k) / 12.0) * (t - r));
  }
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < 512;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    bank[i] = ref_motion[i];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    st->head = 0;
    st->slot_t[0] = 0;
    st->slot_t[1] = 333;
    st->slot_t[2] = 666;
    st->slot_t[3] = -1;
    st->bank_count = 1;
    st->appends = 0;
    st->kv_extra = 0;
    for (int a = 0; a < 4; ++a) st->anchor_fire[a] = 0;
    st->rounds = 0;
    st->frames_in = 0;
    st->frames_out = 0;
    st->initialised = 1;
  }
}

// ------------------------------------------------------------------ ring push
// blockIdx.z = session.
__global__ void ring_push_kernel(DevState* st, float* ring, float* slot_motion,
                                 float* batch_motion, const float* __restrict__ new_noise,
                                 const float* __restrict__ new_motion, int64_t frame_elems) {
  const int z = blockIdx.z;
  st += z;
  ring += z * 16 * frame_elems;
  slot_motion += z * 16 * 512;
  batch_motion += z * 16 * 512;
  new_noise += z * 4 * frame_elems;
  new_motion += z * 4 * 512;
  const int head = st->head;
  const int slot = (head + 3) & 3;
  const int64_t n4 = 4 * frame_elems / 4;
  float4* dst = reinterpret_cast<float4*>(ring + slot * 4 * frame_elems);
  const float4* src = reinterpret_cast<const float4*>(new_noise);
  const int64_t tid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t nthr = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = tid; i < n4; i += nthr) dst[i] = src[i];
  // per-slot motion of the new window, and the batch's motion in batch order
  for (int64_t i = tid; i < 16 * 512; i += nthr) {
    const int f = static_cast<int>(i / 512);
    const int w = f >> 2;
    const int s = (head + w) & 3;
    const int64_t off = (static_cast<int64_t>(s) * 4 + (f & 3)) * 512 + (i % 512);
    float v;
    if (w == 3) {
      v = new_motion[(f & 3) * 512 + (i % 512)];
      slot_motion[off] = v;
    } else {
      v = slot_motion[off];
    }
    batch_motion[i] = v;
  }
  if (tid == 0) {
    if (st->slot_t[slot] != -1) atomicOr(&st->status, DEV_BADARG);
    st->slot_t[slot] = 999;
    st->frames_in += 4;
  }
}

// ------------------------------------------------------------------ DDIM
// Batch frame f = blockIdx.y belongs to window w = f / 4 (oldest first), in
// physical slot (head + w) & 3; blockIdx.z = session. Arithmetic in fp64 (x0
// via the precomputed 1/sqrt(abar_t)), one rounding to fp32 per output.
__global__ void ddim_kernel(const DevState* __restrict__ st, float* ring,
                            const float* __restrict__ eps, float* __restrict__ out_x0,
                            int64_t frame_elems, DdimCoef coef) {
  const int z = blockIdx.z;
  st += z;
  ring += z * 16 * frame_elems;
  eps += z * 16 * frame_elems;
  out_x0 += z * 4 * frame_elems;
  const int f = blockIdx.y;
  const int w = f >> 2, j = f & 3;
  const int slot = (st->head + w) & 3;
  const int ti = t_index(st->slot_t[slot]);
  if (ti < 0) return;
  const double isa = coef.c[ti][0], sb = coef.c[ti][1];
  const double pa = coef.c[ti][2], pb = coef.c[ti][3];
  const int64_t fe4 = frame_elems / 4;
  float4* xf = reinterpret_cast<float4*>(ring) + (static_cast<int64_t>(slot) * 4 + j) * fe4;
  const float4* ef = reinterpret_cast<const float4*>(eps) + static_cast<int64_t>(f) * fe4;
  float4* of = reinterpret_cast<float4*>(out_x0) + static_cast<int64_t>(j) * fe4;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < fe4;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 x = xf[e];
    const float4 ep = ef[e];
    const double x0x = (x.x - sb * ep.x) * isa, x0y = (x.y - sb * ep.y) * isa;
    const double x0z = (x.z - sb * ep.z) * isa, x0w = (x.w - sb * ep.w) * isa;
    if (ti == 3) {
      of[e] = make_float4(static_cast<float>(x0x), static_cast<float>(x0y),
                          static_cast<float>(x0z), static_cast<float>(x0w));
    } else {
      xf[e] = make_float4(static_cast<float>(pa * x0x + pb * ep.x),
                          static_cast<float>(pa * x0y + pb * ep.y),
                          static_cast<float>(pa * x0z + pb * ep.z),
                          static_cast<float>(pa * x0w + pb * ep.w));
    }
  }
}

// one block per session
__global__ void ring_commit_kernel(DevState* st) {
  st += blockIdx.x;
  int popped = 0;
  for (int s = 0; s < 4; ++s) {
    const int t = st->slot_t[s];
    if (t == 0) {
      st->slot_t[s] = -1;
      ++popped;
    } else if (t > 0) {
      st->slot_t[s] = t - 333;
    }
  }
  if (popped != 1) atomicOr(&st->status, DEV_BADARG);
  st->head = (st->head + 1) & 3;
  st->rounds += 1;
  st->frames_out += 4;
}

// ------------------------------------------------------------------ bank check
constexpr int kBankThreads = 256;

__global__ void __launch_bounds__(kBankThreads) bank_check_kernel(
    float* bank, int32_t* count_p, int32_t* appends_p, int capacity, int dim,
    const float* __restrict__ queries, int nq, double thr2, int cap, int32_t* argmin,
    double* min_d2, uint8_t* appended, DevState* st, int count_val) {
  __shared__ double w_best[kBankThreads / 32];
  __shared__ int w_idx[kBankThreads / 32];
  __shared__ int s_cnt, s_app, s_do_append;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nwarps = kBankThreads / 32;
  if (st) {
    // one block per session: its bank, queries, results and state
    const int z = blockIdx.x;
    st += z;
    count_p = &st->bank_count;
    appends_p = &st->appends;
    bank += static_cast<int64_t>(z) * capacity * dim;
    queries += static_cast<int64_t>(z) * nq * dim;
    if (argmin) argmin += z * nq;
    if (min_d2) min_d2 += z * nq;
    if (appended) appended += z * nq;
  }
  if (threadIdx.x == 0) {
    s_cnt = count_p ? *count_p : count_val;
    s_app = appends_p ? *appends_p : 0;
    if (st) {
      for (int a = 0; a < 4; ++a) st->anchor_fire[a] = 0;
    }
  }
  __syncthreads();
  for (int qi = 0; qi < nq; ++qi) {
    const float* q = queries + static_cast<int64_t>(qi) * dim;
    const int cnt = s_cnt;
    double best = INFINITY;
    int bidx = 0x7fffffff;
    for (int j = warp; j < cnt; j += nwarps) {
      const float* b = bank + static_cast<int64_t>(j) * dim;
      double acc = 0.0;
      for (int d = lane; d < dim; d += 32) {
        const double diff = static_cast<double>(q[d]) - static_cast<double>(b[d]);
        acc = fma(diff, diff, acc);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (acc < best) {  // j increases, so the first minimum is kept
        best = acc;
        bidx = j;
      }
    }
    if (lane == 0) {
      w_best[warp] = best;
      w_idx[warp] = bidx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double b = INFINITY;
      int bi = 0x7fffffff;
      for (int w = 0; w < nwarps; ++w) {
        if (w_best[w] < b || (w_best[w] == b && w_idx[w] < bi)) {
          b = w_best[w];
          bi = w_idx[w];
        }
      }
      if (bi == 0x7fffffff) bi = -1;
      if (argmin) argmin[qi] = bi;
      if (min_d2) min_d2[qi] = b;
      const int doit = (cnt > 0 && b > thr2 && s_app < cap && cnt < capacity) ? 1 : 0;
      s_do_append = doit;
      if (appended) appended[qi] = static_cast<uint8_t>(doit);
    }
    __syncthreads();
    if (s_do_append) {
      float* dst = bank + static_cast<int64_t>(cnt) * dim;
      for (int d = threadIdx.x; d < dim; d += kBankThreads) dst[d] = q[d];
      __syncthreads();
      if (threadIdx.x == 0) {
        s_cnt = cnt + 1;
        s_app = s_app + 1;
        if (st && s_app < 4) st->anchor_fire[s_app] = 1;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (count_p) *count_p = s_cnt;
    if (appends_p) *appends_p = s_app;
  }
}

// ------------------------------------------------------------------ motion
struct PeTable {
  float v[32][16];
};

// tok[p][c] = motion[f][16 p + c] + PE[p][c] (fp32);
// kv[f][p][n] = sum_c tok[p][c] * m_kv[c][n] (fp32), n < 2C.
__global__ void motion_kv_kernel(const float* __restrict__ motion, const __half* __restrict__ m_kv,
                                 int C, float* kv, PeTable pe) {
  __shared__ float tok[32][16];
  const int f = blockIdx.y;
  for (int i = threadIdx.x; i < 512; i += blockDim.x) {
    const int p = i >> 4, c = i & 15;
    tok[p][c] = motion[f * 512 + i] + pe.v[p][c];
  }
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= 2 * C) return;
  float w[16];
#pragma unroll
  for (int c = 0; c < 16; ++c) w[c] = __half2float(m_kv[c * 2 * C + n]);
  for (int p = 0; p < 32; ++p) {
    float acc = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) acc = fmaf(tok[p][c], w[c], acc);
    kv[(static_cast<int64_t>(f) * 32 + p) * 2 * C + n] = acc;
  }
}

// One thread per R = 2 query rows (n, n + 128) of one head: R x 32 scores in
// registers, K/V of the frame and head in shared memory (fp32), softmax in
// fp32. Every 16-byte shared-memory read of K or V feeds both rows. Used up
// to head_dim 64 (64x64 layer: whole cross-attention 182 -> 171 us); at
// larger head dims its register cost and halved grid measured slower than
// the one-row kernel below.
constexpr int kMotionRows = 2;

template <int HD>
__global__ void __launch_bounds__(128) motion_attn_kernel(const float* __restrict__ q, int64_t ldq,
                                                          const float* __restrict__ kv, int N,
                                                          int C, __half* __restrict__ out,
                                                          int64_t ldo, float scale) {
  static_assert(HD % 8 == 0, "head_dim");
  constexpr int R = kMotionRows;
  __shared__ __align__(16) float sk[32][HD];
  __shared__ __align__(16) float sv[32][HD];
  const int f = blockIdx.z, h = blockIdx.y;
  const float* kvf = kv + static_cast<int64_t>(f) * 32 * 2 * C;
  for (int i = threadIdx.x; i < 32 * HD; i += blockDim.x) {
    const int p = i / HD, d = i % HD;
    sk[p][d] = kvf[p * 2 * C + h * HD + d];
    sv[p][d] = kvf[p * 2 * C + C + h * HD + d];
  }
  __syncthreads();
  const int n0 = blockIdx.x * 128 * R + threadIdx.x;
  if (n0 >= N) return;
  const float* qr[R];
  bool has[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    has[r] = n0 + 128 * r < N;
    qr[r] = q + (static_cast<int64_t>(f) * N + (has[r] ? n0 + 128 * r : n0)) * ldq + h * HD;
  }
  float s[R][32];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < 32; ++j) s[r][j] = 0.f;
  // the dimension loop stays rolled (a fully unrolled one overflows the
  // instruction cache); the next four dimensions of q are in flight while
  // these are used
  float4 an[R];
#pragma unroll
  for (int r = 0; r < R; ++r) an[r] = *reinterpret_cast<const float4*>(qr[r]);
#pragma unroll 1
  for (int d0 = 0; d0 < HD; d0 += 4) {
    float4 a[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      a[r] = an[r];
      if (d0 + 4 < HD) an[r] = *reinterpret_cast<const float4*>(qr[r] + d0 + 4);
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float4 k = *reinterpret_cast<const float4*>(&sk[j][d0]);
#pragma unroll
      for (int r = 0; r < R; ++r)
        s[r][j] = fmaf(a[r].x, k.x, fmaf(a[r].y, k.y, fmaf(a[r].z, k.z, fmaf(a[r].w, k.w, s[r][j]))));
    }
  }
  float inv[R];
#pragma unroll
  for (int r = 0; r < R; ++r) {
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      s[r][j] *= scale;
      m = fmaxf(m, s[r][j]);
    }
    float l = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      s[r][j] = __expf(s[r][j] - m);
      l += s[r][j];
    }
    inv[r] = 1.f / l;
  }
  __half* orow = out + (static_cast<int64_t>(f) * N + n0) * ldo + h * HD;
#pragma unroll 1
  for (int d0 = 0; d0 < HD; d0 += 8) {
    float o[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[r][e] = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float4 va = *reinterpret_cast<const float4*>(&sv[j][d0]);
      const float4 vb = *reinterpret_cast<const float4*>(&sv[j][d0 + 4]);
      const float v[8] = {va.x, va.y, va.z, va.w, vb.x, vb.y, vb.z, vb.w};
#pragma unroll
      for (int r = 0; r < R; ++r)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[r][e] = fmaf(s[r][j], v[e], o[r][e]);
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (!has[r]) continue;
      uint4 w;
      w.x = pack_half2(o[r][0] * inv[r], o[r][1] * inv[r]);
      w.y = pack_half2(o[r][2] * inv[r], o[r][3] * inv[r]);
      w.z = pack_half2(o[r][4] * inv[r], o[r][5] * inv[r]);
      w.w = pack_half2(o[r][6] * inv[r], o[r][7] * inv[r]);
      *reinterpret_cast<uint4*>(orow + static_cast<int64_t>(128 * r) * ldo + d0) = w;
    }
  }
}

// One thread per (query row, head): 32 scores in registers, smem-resident
// K/V of the frame and head (fp32), softmax in fp32 (head_dim >= 80). The
// dimension loops stay rolled, as in the kernel above.
template <int HD>
__global__ void __launch_bounds__(128) motion_attn_row_kernel(const float* __restrict__ q, int64_t ldq,
                                                          const float* __restrict__ kv, int N,
                                                          int C, __half* __restrict__ out,
                                                          int64_t ldo, float scale) {
  __shared__ float sk[32][HD];
  __shared__ float sv[32][HD];
  const int f = blockIdx.z, h = blockIdx.y;
  const float* kvf = kv + static_cast<int64_t>(f) * 32 * 2 * C;
  for (int i = threadIdx.x; i < 32 * HD; i += blockDim.x) {
    const int p = i / HD, d = i % HD;
    sk[p][d] = kvf[p * 2 * C + h * HD + d];
    sv[p][d] = kvf[p * 2 * C + C + h * HD + d];
  }
  __syncthreads();
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const float* qr = q + (static_cast<int64_t>(f) * N + n) * ldq + h * HD;
  float s[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) s[j] = 0.f;
  float4 qn = *reinterpret_cast<const float4*>(qr);
#pragma unroll 1
  for (int d0 = 0; d0 < HD; d0 += 4) {
    const float4 qv = qn;
    if (d0 + 4 < HD) qn = *reinterpret_cast<const float4*>(qr + d0 + 4);
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      s[j] = fmaf(qv.x, sk[j][d0], s[j]);
      s[j] = fmaf(qv.y, sk[j][d0 + 1], s[j]);
      s[j] = fmaf(qv.z, sk[j][d0 + 2], s[j]);
      s[j] = fmaf(qv.w, sk[j][d0 + 3], s[j]);
    }
  }
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    s[j] *= scale;
    mx = fmaxf(mx, s[j]);
  }
  float sum = 0.f;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    s[j] = __expf(s[j] - mx);
    sum += s[j];
  }
  const float inv = 1.f / sum;
  __half* orow = out + (static_cast<int64_t>(f) * N + n) * ldo + h * HD;
#pragma unroll 1
  for (int d0 = 0; d0 < HD; d0 += 8) {
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = 0.f;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
#pragma unroll
      for (int e = 0; e < 8; ++e) o[e] = fmaf(s[j], sv[j][d0 + e], o[e]);
    }
    uint4 r;
    r.x = pack_half2(o[0] * inv, o[1] * inv);
    r.y = pack_half2(o[2] * inv, o[3] * inv);
    r.z = pack_half2(o[4] * inv, o[5] * inv);
    r.w = pack_half2(o[6] * inv, o[7] * inv);
    *reinterpret_cast<uint4*>(orow + d0) = r;
  }
}

// ------------------------------------------------------------------ nearest (large stores)
// Pass 1: every warp takes whole entries (lanes stride the dimension with
// 16-byte loads); d2 in fp64; each CTA keeps its first minimum and writes it
// to part_d2 / part_idx[blockIdx.x]. Pass 2: one CTA reduces the partials,
// lowest index on equal distances. One read of the store in total.
constexpr int kNearThreads = 256;

__global__ void __launch_bounds__(kNearThreads) nearest_partial_kernel(
    const float* __restrict__ store, int64_t count, int dim, const float* __restrict__ query,
    double* part_d2, int64_t* part_idx) {
  __shared__ double w_best[kNearThreads / 32];
  __shared__ int64_t w_idx[kNearThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (kNearThreads / 32) + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (kNearThreads / 32);
  double best = INFINITY;
  int64_t bidx = INT64_MAX;
  const bool vec = (dim % 4) == 0 && dim <= 128;
  constexpr int U = 4;   // entries per warp iteration (more loads in flight)
  for (int64_t j0 = gw * U; j0 < count; j0 += nw * U) {
    double acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = 0.0;
    if (vec) {
      // dim <= 128: one 16-byte chunk per lane and entry
      const int d = 4 * lane;
      float4 a[U];
      float4 q = make_float4(0.f, 0.f, 0.f, 0.f);
      if (d < dim) q = *reinterpret_cast<const float4*>(query + d);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        a[u] = q;   // entries past the end contribute nothing
        if (d < dim && j0 + u < count)
          a[u] = *reinterpret_cast<const float4*>(store + (j0 + u) * dim + d);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const double d0 = static_cast<double>(q.x) - a[u].x, d1 = static_cast<double>(q.y) - a[u].y;
        const double d2 = static_cast<double>(q.z) - a[u].z, d3 = static_cast<double>(q.w) - a[u].w;
        acc[u] = fma(d3, d3, fma(d2, d2, fma(d1, d1, d0 * d0)));
      }
    } else {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (j0 + u >= count) continue;
        const float* e = store + (j0 + u) * dim;
        for (int d = lane; d < dim; d += 32) {
          const double df = static_cast<double>(query[d]) - e[d];
          acc[u] = fma(df, df, acc[u]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
      for (int u = 0; u < U; ++u) acc[u] += __shfl_xor_sync(0xffffffffu, acc[u], o);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (j0 + u < count && acc[u] < best) {   // entries of a warp increase
        best = acc[u];
        bidx = j0 + u;
      }
    }
  }
  if (lane == 0) {
    w_best[warp] = best;
    w_idx[warp] = bidx;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double b = INFINITY;
    int64_t bi = INT64_MAX;
    for (int w = 0; w < kNearThreads / 32; ++w)
      if (w_best[w] < b || (w_best[w] == b && w_idx[w] < bi)) {
        b = w_best[w];
        bi = w_idx[w];
      }
    part_d2[blockIdx.x] = b;
    part_idx[blockIdx.x] = bi;
  }
}

__global__ void nearest_reduce_kernel(const double* part_d2, const int64_t* part_idx, int parts,
                                      int64_t* argmin, double* min_d2) {
  __shared__ double sb[256];
  __shared__ int64_t si[256];
  double b = INFINITY;
  int64_t bi = INT64_MAX;
  for (int k = threadIdx.x; k < parts; k += blockDim.x)
    if (part_d2[k] < b || (part_d2[k] == b && part_idx[k] < bi)) {
      b = part_d2[k];
      bi = part_idx[k];
    }
  sb[threadIdx.x] = b;
  si[threadIdx.x] = bi;
  __syncthreads();
  for (int o = blockDim.x / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      const double ob = sb[threadIdx.x + o];
      const int64_t oi = si[threadIdx.x + o];
      if (ob < sb[threadIdx.x] || (ob == sb[threadIdx.x] && oi < si[threadIdx.x])) {
        sb[threadIdx.x] = ob;
        si[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *argmin = si[0] == INT64_MAX ? -1 : si[0];
    if (min_d2) *min_d2 = sb[0];
  }
}

int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = 148 * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_prefill(DevState* st, float* ring, float* slot_motion, float* bank,
                           const float* ref_latent, const float* prefill_eps,
                           const float* ref_motion, const float* drive0, int64_t frame_elems,
                           int capacity, int sessions, cudaStream_t s) {
  DdimCoef coef;
  ddim_coefficients(&coef);
  const dim3 grid(static_cast<unsigned>(grid_for(12 * frame_elems, 256)), 1, sessions);
  prefill_kernel<<<grid, 256, 0, s>>>(st, ring, slot_motion, bank, ref_latent, prefill_eps,
                                      ref_motion, drive0, frame_elems, capacity, coef);
  return cudaGetLastError();
}

cudaError_t launch_ring_push(DevState* st, float* ring, float* slot_motion, float* batch_motion,
                             const float* new_noise, const float* new_motion,
                             int64_t frame_elems, int sessions, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(grid_for(frame_elems, 256)), 1, sessions);
  ring_push_kernel<<<grid, 256, 0, s>>>(st, ring, slot_motion, batch_motion, new_noise, new_motion,
                                        frame_elems);
  return cudaGetLastError();
}

cudaError_t launch_ddim(DevState* st, float* ring, const float* eps, float* out_x0,
                        int64_t frame_elems, const DdimCoef& coef, int sessions, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>((grid_for(frame_elems / 4, 256) + 15) / 16), 16, sessions);
  ddim_kernel<<<grid, 256, 0, s>>>(st, ring, eps, out_x0, frame_elems, coef);
  return cudaGetLastError();
}

cudaError_t launch_ring_commit(DevState* st, int sessions, cudaStream_t s) {
  ring_commit_kernel<<<sessions, 1, 0, s>>>(st);
  return cudaGetLastError();
}

cudaError_t launch_bank_check(float* bank, int32_t* count, int32_t* appends, int capacity,
                              int dim, const float* queries, int nq, double thr2, int cap,
                              int32_t* argmin, double* min_d2, uint8_t* appended,
                              DevState* st, int sessions, cudaStream_t s) {
  if (!st && sessions != 1) return cudaErrorInvalidValue;
  bank_check_kernel<<<sessions, kBankThreads, 0, s>>>(bank, count, appends, capacity, dim, queries,
                                                      nq, thr2, cap, argmin, min_d2, appended, st,
                                                      0);
  return cudaGetLastError();
}

cudaError_t launch_nearest(const float* store, int count, int dim, const float* query,
                           int32_t* argmin, double* min_d2, cudaStream_t s) {
  // a bank check with no append allowed: the nearest stored vector
  bank_check_kernel<<<1, kBankThreads, 0, s>>>(const_cast<float*>(store), nullptr, nullptr, count,
                                               dim, query, 1, 0.0, 0, argmin, min_d2, nullptr,
                                               nullptr, count);
  return cudaGetLastError();
}

int nearest_parts(int64_t count) {
  int64_t g = (count + (kNearThreads / 32) * 4 - 1) / ((kNearThreads / 32) * 4);
  if (g > 148 * 8) g = 148 * 8;
  return static_cast<int>(g < 1 ? 1 : g);
}

cudaError_t launch_nearest_large(const float* store, int64_t count, int dim, const float* query,
                                 double* part_d2, int64_t* part_idx, int parts, int64_t* argmin,
                                 double* min_d2, cudaStream_t s) {
  nearest_partial_kernel<<<parts, kNearThreads, 0, s>>>(store, count, dim, query, part_d2,
                                                        part_idx);
  nearest_reduce_kernel<<<1, 256, 0, s>>>(part_d2, part_idx, parts, argmin, min_d2);
  return cudaGetLastError();
}

cudaError_t launch_motion_kv(const float* motion, const __half* m_kv, int F, int C, float* kv,
                             cudaStream_t s) {
  PeTable pe;
  for (int p = 0; p < 32; ++p)
    for (int i = 0; i < 8; ++i) {
      const double ang = p / std::pow(10000.0, 2.0 * i / 16.0);
      pe.v[p][2 * i] = static_cast<float>(std::sin(ang));
      pe.v[p][2 * i + 1] = static_cast<float>(std::cos(ang));
    }
  dim3 grid((2 * C + 255) / 256, F);
  motion_kv_kernel<<<grid, 256, 0, s>>>(motion, m_kv, C, kv, pe);
  return cudaGetLastError();
}

cudaError_t launch_motion_attn(const float* q, int64_t ldq, const float* kv, int F, int N,
                               int C, int heads, __half* out, int64_t ldo, cudaStream_t s) {
  const int hd = C / heads;
  const float scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(hd)));
  auto grid = [&](int rows) { return dim3((N + 128 * rows - 1) / (128 * rows), heads, F); };
  switch (hd) {
    case 40: motion_attn_kernel<40><<<grid(kMotionRows), 128, 0, s>>>(q, ldq, kv, N, C, out, ldo, scale); break;
    case 64: motion_attn_kernel<64><<<grid(kMotionRows), 128, 0, s>>>(q, ldq, kv, N, C, out, ldo, scale); break;
    case 80: motion_attn_row_kernel<80><<<grid(1), 128, 0, s>>>(q, ldq, kv, N, C, out, ldo, scale); break;
    case 128: motion_attn_row_kernel<128><<<grid(1), 128, 0, s>>>(q, ldq, kv, N, C, out, ldo, scale); break;
    case 160: motion_attn_row_kernel<160><<<grid(1), 128, 0, s>>>(q, ldq, kv, N, C, out, ldo, scale); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pl
