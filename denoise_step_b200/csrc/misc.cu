#include <cmath>

#include "devinit.cuh"
#include "fastmath.cuh"
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
// In-order bank check ([PL] 抗身份漂移的补丁): query k sees the stored entries
// and the queries appended before it in the same call. An appended entry is
// the query itself, bit for bit, so every distance the check can need is one
// of two kinds, both fixed before any decision: query k to a stored entry j,
// and query k to an earlier query i. They are computed in one parallel pass
// (fp64 from the fp32 values, one warp per pair or per entry); the decisions
// then run in order over that table: nearest stored entry (lowest index on
// ties), then the earlier appended queries in their append order (their bank
// indices follow the stored ones); append when d^2 > thr^2, the cap allows
// it and the bank has room.
constexpr int kBankThreads = 256;
constexpr int kBankSmall = 32;     // capacity and queries of the one-CTA path

// squared distance of two fp32 vectors in fp64, summed over the warp (every
// lane gets the total)
__device__ __forceinline__ double dist2_warp(const float* a, const float* b, int dim, int lane) {
  double acc = 0.0;
  const bool vec = (dim & 3) == 0 &&
                   ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 15) == 0;
  if (vec) {
    for (int d = 4 * lane; d < dim; d += 128) {
      const float4 x = *reinterpret_cast<const float4*>(a + d);
      const float4 y = *reinterpret_cast<const float4*>(b + d);
      const double d0 = static_cast<double>(x.x) - y.x, d1 = static_cast<double>(x.y) - y.y;
      const double d2 = static_cast<double>(x.z) - y.z, d3 = static_cast<double>(x.w) - y.w;
      acc = fma(d3, d3, fma(d2, d2, fma(d1, d1, fma(d0, d0, acc))));
    }
  } else {
    for (int d = lane; d < dim; d += 32) {
      const double df = static_cast<double>(a[d]) - b[d];
      acc = fma(df, df, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Decisions of one call, in query order, from the existing-entry minima (per
// query: d2 and index, index -1 when the bank is empty) and the query-query
// table dq[k * ldq + i] (i < k). Run by one thread. Returns the appends made;
// list[a] = query appended a-th.
__device__ int bank_decide(const double* e_d2, const int* e_idx, const double* dq, int ldq,
                           int nq, int cnt0, int app0, int capacity, double thr2, int cap,
                           int32_t* argmin, double* min_d2, uint8_t* appended, int* list,
                           DevState* st) {
  int cnt = cnt0, app = app0, n_app = 0;
  for (int k = 0; k < nq; ++k) {
    double best = e_d2[k];
    int bi = e_idx[k];
    for (int a = 0; a < n_app; ++a) {
      const double d = dq[k * ldq + list[a]];
      if (d < best) {   // appended entries come after the stored ones
        best = d;
        bi = cnt0 + a;
      }
    }
    if (argmin) argmin[k] = bi;
    if (min_d2) min_d2[k] = best;
    const bool doit = cnt > 0 && best > thr2 && app < cap && cnt < capacity;
    if (appended) appended[k] = doit ? 1 : 0;
    if (doit) {
      list[n_app++] = k;
      ++cnt;
      ++app;
      if (st && app < 4) st->anchor_fire[app] = 1;
    }
  }
  return n_app;
}

// One CTA per session (the round's check; capacity and queries <= kBankSmall).
__global__ void __launch_bounds__(kBankThreads) bank_check_kernel(
    float* bank, int32_t* count_p, int32_t* appends_p, int capacity, int dim,
    const float* __restrict__ queries, int nq, double thr2, int cap, int32_t* argmin,
    double* min_d2, uint8_t* appended, DevState* st) {
  __shared__ double s_de[kBankSmall * kBankSmall];   // [k][j]: query k, stored entry j
  __shared__ double s_dq[kBankSmall * kBankSmall];   // [k][i]: query k, earlier query i
  __shared__ double s_bd[kBankSmall];
  __shared__ int s_bi[kBankSmall], s_list[kBankSmall];
  __shared__ int s_cnt0, s_app0, s_napp;
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
    int c = *count_p;
    s_cnt0 = c < 0 ? 0 : (c > capacity ? capacity : c);
    s_app0 = *appends_p;
    if (st)
      for (int a = 0; a < 4; ++a) st->anchor_fire[a] = 0;
  }
  __syncthreads();
  const int cnt0 = s_cnt0;
  const int n_e = nq * cnt0, n_all = n_e + nq * nq;
  for (int p = warp; p < n_all; p += nwarps) {
    int k, j;
    const float* b;
    if (p < n_e) {
      k = p / cnt0;
      j = p - k * cnt0;
      b = bank + static_cast<int64_t>(j) * dim;
    } else {
      k = (p - n_e) / nq;
      j = (p - n_e) - k * nq;
      if (j >= k) continue;   // warp-uniform
      b = queries + static_cast<int64_t>(j) * dim;
    }
    const double d = dist2_warp(queries + static_cast<int64_t>(k) * dim, b, dim, lane);
    if (lane == 0) (p < n_e ? s_de : s_dq)[k * kBankSmall + j] = d;
  }
  __syncthreads();
  if (threadIdx.x < nq) {
    // nearest stored entry of query threadIdx.x (ascending j, strict <)
    const int k = threadIdx.x;
    double b = INFINITY;
    int bi = -1;
    for (int j = 0; j < cnt0; ++j)
      if (s_de[k * kBankSmall + j] < b) {
        b = s_de[k * kBankSmall + j];
        bi = j;
      }
    s_bd[k] = b;
    s_bi[k] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int n_app = bank_decide(s_bd, s_bi, s_dq, kBankSmall, nq, cnt0, s_app0, capacity, thr2,
                                  cap, argmin, min_d2, appended, s_list, st);
    s_napp = n_app;
    *count_p = cnt0 + n_app;
    *appends_p = s_app0 + n_app;
  }
  __syncthreads();
  for (int a = 0; a < s_napp; ++a) {
    const float* src = queries + static_cast<int64_t>(s_list[a]) * dim;
    float* dst = bank + static_cast<int64_t>(cnt0 + a) * dim;
    for (int d = threadIdx.x; d < dim; d += kBankThreads) dst[d] = src[d];
  }
}

// Large banks, pass 1: each CTA takes a slice of the stored entries and keeps,
// per query, its nearest entry (lowest index on ties). Every entry is read
// once for all queries; the queries sit in shared memory as fp64. Four lanes
// share an entry: each lane walks its quarter of the row in 16-byte chunks,
// so a warp load covers 8 rows x 64 contiguous bytes (whole sectors), the
// four lanes of an entry read different query values and the eight entries
// the same ones (broadcast, no bank conflict), and an entry's sum needs two
// shuffle steps. Each lane takes kBankE entries at once (slot + 8 e), so a
// query value read from shared memory serves kBankE entries: with one it
// was the shared-memory reads that bound the pass (L1 pipe 82%). Measured
// alternatives at 262144 x 512 with 4 queries: a warp per entry (five-step
// reduction per entry and query, 124 registers) and a thread per entry (32
// rows per warp load, L1-bound at 93%) both ran at ~2.2 TB/s.
constexpr int kBankGroup = 4;
constexpr int kBankLanes = 4;              // lanes per entry
constexpr int kBankE = 4;                  // entries per lane at once (2 measured slower)
constexpr int kBankMaxQueries = 64;

__global__ void __launch_bounds__(kBankThreads) bank_partial_kernel(
    const float* __restrict__ bank, const int32_t* count_p, int64_t capacity, int dim,
    const float* __restrict__ queries, int nq, double* part_d2, int64_t* part_idx,
    const int32_t* need) {
  extern __shared__ double sq[];                    // [nq][dim]
  // run only when the fp32 screen left a query undecided
  if (need != nullptr && *((volatile const int32_t*)need) == 0) return;
  __shared__ double w_best[kBankThreads / 32][kBankMaxQueries];
  __shared__ int64_t w_idx[kBankThreads / 32][kBankMaxQueries];
  constexpr int kSlots = 32 / kBankLanes;
  constexpr int kPerWarp = kSlots * kBankE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % kBankLanes, slot = lane / kBankLanes;
  for (int i = threadIdx.x; i < nq * dim; i += kBankThreads) sq[i] = static_cast<double>(queries[i]);
  __syncthreads();
  int64_t cnt = *count_p;
  cnt = cnt < 0 ? 0 : (cnt > capacity ? capacity : cnt);
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (kBankThreads / 32) + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (kBankThreads / 32);
  const bool vec = (dim & 3) == 0 && (reinterpret_cast<uintptr_t>(bank) & 15) == 0;
  for (int g0 = 0; g0 < nq; g0 += kBankGroup) {
    const int gn = nq - g0 < kBankGroup ? nq - g0 : kBankGroup;
    const double* q0 = sq + static_cast<int64_t>(g0) * dim;
    double best[kBankGroup];
    int64_t bidx[kBankGroup];
#pragma unroll
    for (int g = 0; g < kBankGroup; ++g) {
      best[g] = INFINITY;
      bidx[g] = -1;
    }
    for (int64_t j0 = gw * kPerWarp; j0 < cnt; j0 += nw * kPerWarp) {
      // a lane's entries: j0 + slot + kSlots * u, increasing
      double acc[kBankE][kBankGroup];
#pragma unroll
      for (int u = 0; u < kBankE; ++u)
#pragma unroll
        for (int g = 0; g < kBankGroup; ++g) acc[u][g] = 0.0;
      const float* e[kBankE];
      bool ok[kBankE];
#pragma unroll
      for (int u = 0; u < kBankE; ++u) {
        const int64_t j = j0 + slot + kSlots * u;
        ok[u] = j < cnt;
        e[u] = bank + (ok[u] ? j : 0) * dim;   // rows past the end read row 0, unused
      }
      if (vec) {
#pragma unroll 2
        for (int d = 4 * sub; d < dim; d += 4 * kBankLanes) {
          double x[kBankE][4];
#pragma unroll
          for (int u = 0; u < kBankE; ++u) {
            const float4 t = __ldg(reinterpret_cast<const float4*>(e[u] + d));
            x[u][0] = t.x;
            x[u][1] = t.y;
            x[u][2] = t.z;
            x[u][3] = t.w;
          }
#pragma unroll
          for (int g = 0; g < kBankGroup; ++g) {
            if (g < gn) {
              const double2 qa = *reinterpret_cast<const double2*>(q0 + g * dim + d);
              const double2 qb = *reinterpret_cast<const double2*>(q0 + g * dim + d + 2);
#pragma unroll
              for (int u = 0; u < kBankE; ++u) {
                const double d0 = qa.x - x[u][0], d1 = qa.y - x[u][1];
                const double d2 = qb.x - x[u][2], d3 = qb.y - x[u][3];
                acc[u][g] = fma(d3, d3, fma(d2, d2, fma(d1, d1, fma(d0, d0, acc[u][g]))));
              }
            }
          }
        }
      } else {
        for (int d = sub; d < dim; d += kBankLanes) {
          double x[kBankE];
#pragma unroll
          for (int u = 0; u < kBankE; ++u) x[u] = e[u][d];
#pragma unroll
          for (int g = 0; g < kBankGroup; ++g)
            if (g < gn) {
              const double q = q0[g * dim + d];
#pragma unroll
              for (int u = 0; u < kBankE; ++u) {
                const double df = q - x[u];
                acc[u][g] = fma(df, df, acc[u][g]);
              }
            }
        }
      }
#pragma unroll
      for (int u = 0; u < kBankE; ++u) {
#pragma unroll
        for (int g = 0; g < kBankGroup; ++g) {
          if (g < gn) {
#pragma unroll
            for (int o = 1; o < kBankLanes; o <<= 1)
              acc[u][g] += __shfl_xor_sync(0xffffffffu, acc[u][g], o);
            if (ok[u] && acc[u][g] < best[g]) {
              best[g] = acc[u][g];
              bidx[g] = j0 + slot + kSlots * u;
            }
          }
        }
      }
    }
    // warp minimum per query (lowest index on ties), then one entry per warp
#pragma unroll
    for (int g = 0; g < kBankGroup; ++g) {
      if (g < gn) {
        double b = best[g];
        int64_t bi = bidx[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const double ob = __shfl_xor_sync(0xffffffffu, b, o);
          const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
          if (oi >= 0 && (bi < 0 || ob < b || (ob == b && oi < bi))) {
            b = ob;
            bi = oi;
          }
        }
        if (lane == 0) {
          w_best[warp][g0 + g] = b;
          w_idx[warp][g0 + g] = bi;
        }
      }
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nq; k += kBankThreads) {
    double b = INFINITY;
    int64_t bi = -1;
    for (int w = 0; w < kBankThreads / 32; ++w) {
      const int64_t wi = w_idx[w][k];
      if (wi >= 0 && (bi < 0 || w_best[w][k] < b || (w_best[w][k] == b && wi < bi))) {
        b = w_best[w][k];
        bi = wi;
      }
    }
    part_d2[static_cast<int64_t>(blockIdx.x) * nq + k] = b;
    part_idx[static_cast<int64_t>(blockIdx.x) * nq + k] = bi;
  }
}

// Large banks, fp32 screen: the traversal of the fp64 pass (four lanes per
// entry, each walking its quarter of the row in 16-byte chunks; queries in
// shared memory) with fp32 arithmetic, which needs half the registers: three
// CTAs per SM instead of two, so more rows in flight (the fp64 pass and this
// one are bound by the loads in flight, not by their arithmetic: at 262144 x
// 512 with 4 queries, fp32 with two CTAs per SM ran as fast as fp64, a warp per
// row with the queries in registers (one CTA per SM) 45% slower, and eight
// entries per lane (one CTA per SM) 10% slower). Per query it keeps the smallest
// computed d^2 (its index, lowest on ties) and the second smallest. Rounding
// bound: each lane sums its n = dim / 4 terms (q - x)^2 with one fma per term,
// the subtraction rounded once, and two shuffle additions join the lanes, so
// the computed value is within (n + 4) u of the exact d^2, relative (u =
// 2^-24, all terms non-negative): 132 u ~ 7.9e-6 at dim 512. When the second
// smallest exceeds the smallest by more than twice that bound, the smallest
// is the exact argmin and the fp64 pass is not needed; bank_select_kernel
// asks for a gap of 4e-5 (a 2.5x margin at dim 512), scaled with n past it.
__device__ __forceinline__ void top2_push(float c, int64_t j, float& b1, int64_t& i1, float& b2) {
  if (c < b1) {
    b2 = b1;
    b1 = c;
    i1 = j;
  } else if (c < b2) {
    b2 = c;
  }
}
// merge (o1, oi, o2) into (b1, i1, b2): lowest index first on equal values;
// the same entry seen twice (the lanes that share an entry all hold its sum)
// counts once
__device__ __forceinline__ void top2_merge(float& b1, int64_t& i1, float& b2, float o1, int64_t oi,
                                           float o2) {
  if (oi < 0) return;
  if (oi == i1) {
    b2 = fminf(b2, o2);
    return;
  }
  if (i1 < 0 || o1 < b1 || (o1 == b1 && oi < i1)) {
    b2 = fminf(b1, o2);
    b1 = o1;
    i1 = oi;
  } else {
    b2 = fminf(b2, o1);
  }
}

constexpr int kScreenE = 4;        // entries per lane at once
constexpr int kScreenBlocks = 3;   // CTAs per SM (80 registers a thread)

__global__ void __launch_bounds__(kBankThreads, kScreenBlocks) bank_screen_kernel(
    const float* __restrict__ bank, const int32_t* count_p, int64_t capacity, int dim,
    const float* __restrict__ queries, int nq, float* part_b1, int64_t* part_i1, float* part_b2) {
  extern __shared__ float sqf[];                    // [nq][dim]
  __shared__ float w_b1[kBankThreads / 32][kBankMaxQueries];
  __shared__ float w_b2[kBankThreads / 32][kBankMaxQueries];
  __shared__ int64_t w_i1[kBankThreads / 32][kBankMaxQueries];
  constexpr int kSlots = 32 / kBankLanes;
  constexpr int kPerWarp = kSlots * kScreenE;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % kBankLanes, slot = lane / kBankLanes;
  for (int i = threadIdx.x; i < nq * dim; i += kBankThreads) sqf[i] = queries[i];
  __syncthreads();
  int64_t cnt = *count_p;
  cnt = cnt < 0 ? 0 : (cnt > capacity ? capacity : cnt);
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * (kBankThreads / 32) + warp;
  const int64_t nw = static_cast<int64_t>(gridDim.x) * (kBankThreads / 32);
  for (int g0 = 0; g0 < nq; g0 += kBankGroup) {
    const int gn = nq - g0 < kBankGroup ? nq - g0 : kBankGroup;
    const float* q0 = sqf + static_cast<int64_t>(g0) * dim;
    float b1[kBankGroup], b2[kBankGroup];
    int64_t i1[kBankGroup];
#pragma unroll
    for (int g = 0; g < kBankGroup; ++g) {
      b1[g] = INFINITY;
      b2[g] = INFINITY;
      i1[g] = -1;
    }
    for (int64_t j0 = gw * kPerWarp; j0 < cnt; j0 += nw * kPerWarp) {
      // a lane's entries: j0 + slot + kSlots * u, increasing
      float acc[kScreenE][kBankGroup];
#pragma unroll
      for (int u = 0; u < kScreenE; ++u)
#pragma unroll
        for (int g = 0; g < kBankGroup; ++g) acc[u][g] = 0.f;
      const float* e[kScreenE];
      bool ok[kScreenE];
#pragma unroll
      for (int u = 0; u < kScreenE; ++u) {
        const int64_t j = j0 + slot + kSlots * u;
        ok[u] = j < cnt;
        e[u] = bank + (ok[u] ? j : 0) * dim;   // rows past the end read row 0, unused
      }
      for (int d = 4 * sub; d < dim; d += 4 * kBankLanes) {
        float4 x[kScreenE];
#pragma unroll
        for (int u = 0; u < kScreenE; ++u) x[u] = __ldg(reinterpret_cast<const float4*>(e[u] + d));
#pragma unroll
        for (int g = 0; g < kBankGroup; ++g) {
          if (g < gn) {
            const float4 q = *reinterpret_cast<const float4*>(q0 + g * dim + d);
#pragma unroll
            for (int u = 0; u < kScreenE; ++u) {
              const float d0 = q.x - x[u].x, d1 = q.y - x[u].y;
              const float d2 = q.z - x[u].z, d3 = q.w - x[u].w;
              acc[u][g] = fmaf(d3, d3, fmaf(d2, d2, fmaf(d1, d1, fmaf(d0, d0, acc[u][g]))));
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kScreenE; ++u) {
#pragma unroll
        for (int g = 0; g < kBankGroup; ++g) {
          if (g < gn) {
#pragma unroll
            for (int o = 1; o < kBankLanes; o <<= 1)
              acc[u][g] += __shfl_xor_sync(0xffffffffu, acc[u][g], o);
            if (ok[u]) top2_push(acc[u][g], j0 + slot + kSlots * u, b1[g], i1[g], b2[g]);
          }
        }
      }
    }
    // warp state per query: the lanes of an entry hold the same candidates,
    // which the merge counts once
#pragma unroll
    for (int g = 0; g < kBankGroup; ++g) {
      if (g < gn) {
        float a1 = b1[g], a2 = b2[g];
        int64_t ai = i1[g];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          const float o1 = __shfl_xor_sync(0xffffffffu, a1, o);
          const float o2 = __shfl_xor_sync(0xffffffffu, a2, o);
          const int64_t oi = __shfl_xor_sync(0xffffffffu, ai, o);
          top2_merge(a1, ai, a2, o1, oi, o2);
        }
        if (lane == 0) {
          w_b1[warp][g0 + g] = a1;
          w_b2[warp][g0 + g] = a2;
          w_i1[warp][g0 + g] = ai;
        }
      }
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < nq; k += kBankThreads) {
    float a1 = INFINITY, a2 = INFINITY;
    int64_t ai = -1;
    for (int w = 0; w < kBankThreads / 32; ++w) top2_merge(a1, ai, a2, w_b1[w][k], w_i1[w][k], w_b2[w][k]);
    const int64_t o = static_cast<int64_t>(blockIdx.x) * nq + k;
    part_b1[o] = a1;
    part_b2[o] = a2;
    part_i1[o] = ai;
  }
}

// the screen's layout: rows of a multiple of 4 floats, 16-byte aligned
bool bank_screen_ok(int dim, const float* bank, const float* queries) {
  return dim % 4 == 0 &&
         ((reinterpret_cast<uintptr_t>(bank) | reinterpret_cast<uintptr_t>(queries)) & 15) == 0;
}

constexpr float kBankScreenGap = 4e-5f;

// Large banks, screen decision (one CTA): per query the screen's nearest entry
// and whether it is certain; need = 1 when any query needs the fp64 pass.
__global__ void set_flag_kernel(int32_t* flag, int32_t v) { *flag = v; }

__global__ void __launch_bounds__(kBankThreads) bank_select_kernel(
    const int32_t* count_p, int64_t capacity, int dim, int nq, const float* part_b1,
    const int64_t* part_i1, const float* part_b2, int parts, int64_t* sel_idx, int32_t* need) {
  __shared__ int s_need;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) s_need = 0;
  __syncthreads();
  int64_t cnt = *count_p;
  cnt = cnt < 0 ? 0 : (cnt > capacity ? capacity : cnt);
  // twice the rounding bound (n + 4) u with a 2.5x margin, n = dim / 4
  const float gap = kBankScreenGap * fmaxf(1.0f, (dim / kBankLanes + 4) / 132.0f);
  for (int k = warp; k < nq; k += kBankThreads / 32) {
    float a1 = INFINITY, a2 = INFINITY;
    int64_t ai = -1;
    // eight partials per lane loaded before any is merged (one load latency
    // per batch, not per partial)
    for (int p0 = 0; p0 < parts; p0 += 8 * 32) {
      float l1[8], l2[8];
      int64_t li[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int pt = p0 + r * 32 + lane;
        const int64_t o = static_cast<int64_t>(pt < parts ? pt : 0) * nq + k;
        l1[r] = part_b1[o];
        l2[r] = part_b2[o];
        li[r] = pt < parts ? part_i1[o] : -1;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) top2_merge(a1, ai, a2, l1[r], li[r], l2[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float o1 = __shfl_xor_sync(0xffffffffu, a1, o);
      const float o2 = __shfl_xor_sync(0xffffffffu, a2, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, ai, o);
      top2_merge(a1, ai, a2, o1, oi, o2);
    }
    if (lane == 0) {
      // certain: no entry; or a candidate that is the only entry or leads
      // the runner-up by a finite gap past the rounding bound (an overflow to
      // infinity, a NaN or a near-zero pair leaves the query to the fp64 pass)
      const bool certain =
          cnt == 0 || (ai >= 0 && (cnt == 1 || (a2 < INFINITY && a2 > 1e-20f && a2 - a1 > gap * a2)));
      sel_idx[k] = cnt == 0 ? -1 : ai;
      if (!certain) atomicOr(&s_need, 1);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) *need = s_need;
}

// Large banks, pass 2 (one CTA): per query the minimum over the partial
// minima, the query-query distances, the in-order decisions and the copies.
__global__ void __launch_bounds__(kBankThreads) bank_resolve_kernel(
    float* bank, int32_t* count_p, int32_t* appends_p, int capacity, int dim,
    const float* __restrict__ queries, int nq, double thr2, int cap, const double* part_d2,
    const int64_t* part_idx, int parts, const int64_t* sel_idx, const int32_t* need,
    int32_t* argmin, double* min_d2, uint8_t* appended) {
  __shared__ double s_dq[kBankMaxQueries * kBankMaxQueries];
  __shared__ double s_bd[kBankMaxQueries];
  __shared__ int s_bi[kBankMaxQueries], s_list[kBankMaxQueries];
  __shared__ int s_cnt0, s_app0, s_napp;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int nwarps = kBankThreads / 32;
  if (threadIdx.x == 0) {
    const int c = *count_p;
    s_cnt0 = c < 0 ? 0 : (c > capacity ? capacity : c);
    s_app0 = *appends_p;
  }
  const bool screened = need != nullptr && *((volatile const int32_t*)need) == 0;
  if (screened) {
    // the screen fixed every nearest stored entry: its exact fp64 d^2
    for (int k = warp; k < nq; k += nwarps) {
      const int64_t j = sel_idx[k];
      const double d = j >= 0 ? dist2_warp(queries + static_cast<int64_t>(k) * dim,
                                           bank + j * static_cast<int64_t>(dim), dim, lane)
                              : INFINITY;
      if (lane == 0) {
        s_bd[k] = d;
        s_bi[k] = static_cast<int>(j);
      }
    }
  }
  // per query: one warp reduces the partial minima (lowest index on ties)
  for (int k = warp; !screened && k < nq; k += nwarps) {
    double b = INFINITY;
    int64_t bi = -1;
    for (int pt = lane; pt < parts; pt += 32) {
      const double d = part_d2[static_cast<int64_t>(pt) * nq + k];
      const int64_t i = part_idx[static_cast<int64_t>(pt) * nq + k];
      if (i >= 0 && (d < b || (d == b && (bi < 0 || i < bi)))) {
        b = d;
        bi = i;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ob = __shfl_xor_sync(0xffffffffu, b, o);
      const int64_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (oi >= 0 && (bi < 0 || ob < b || (ob == b && oi < bi))) {
        b = ob;
        bi = oi;
      }
    }
    if (lane == 0) {
      s_bd[k] = b;
      s_bi[k] = static_cast<int>(bi);
    }
  }
  // query-query distances (i < k)
  for (int p = warp; p < nq * nq; p += nwarps) {
    const int k = p / nq, i = p - (p / nq) * nq;
    if (i >= k) continue;   // warp-uniform
    const double d = dist2_warp(queries + static_cast<int64_t>(k) * dim,
                                queries + static_cast<int64_t>(i) * dim, dim, lane);
    if (lane == 0) s_dq[k * kBankMaxQueries + i] = d;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int n_app = bank_decide(s_bd, s_bi, s_dq, kBankMaxQueries, nq, s_cnt0, s_app0, capacity,
                                  thr2, cap, argmin, min_d2, appended, s_list, nullptr);
    s_napp = n_app;
    *count_p = s_cnt0 + n_app;
    *appends_p = s_app0 + n_app;
  }
  __syncthreads();
  for (int a = 0; a < s_napp; ++a) {
    const float* src = queries + static_cast<int64_t>(s_list[a]) * dim;
    float* dst = bank + static_cast<int64_t>(s_cnt0 + a) * dim;
    for (int d = threadIdx.x; d < dim; d += kBankThreads) dst[d] = src[d];
  }
}

// Nearest of `count` stored vectors to one query (pose retrieval), one CTA.
__global__ void __launch_bounds__(kBankThreads) nearest_small_kernel(
    const float* __restrict__ store, int count, int dim, const float* __restrict__ query,
    int32_t* argmin, double* min_d2) {
  __shared__ double w_best[kBankThreads / 32];
  __shared__ int w_idx[kBankThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  double best = INFINITY;
  int bidx = -1;
  for (int j = warp; j < count; j += kBankThreads / 32) {
    const double d = dist2_warp(query, store + static_cast<int64_t>(j) * dim, dim, lane);
    if (d < best) {   // a warp's entries increase
      best = d;
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
    int bi = -1;
    for (int w = 0; w < kBankThreads / 32; ++w)
      if (w_idx[w] >= 0 && (w_best[w] < b || (w_best[w] == b && w_idx[w] < bi))) {
        b = w_best[w];
        bi = w_idx[w];
      }
    *argmin = bi;
    if (min_d2) *min_d2 = b;
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

int bank_parts(int64_t capacity) {
  constexpr int kEntriesPerCta = kBankThreads / kBankLanes * kBankE;
  int64_t g = (capacity + kEntriesPerCta - 1) / kEntriesPerCta;
  if (g > 148 * 8) g = 148 * 8;
  return static_cast<int>(g < 1 ? 1 : g);
}

bool bank_small(int capacity, int nq) { return capacity <= kBankSmall && nq <= kBankSmall; }

// large-path workspace: fp64 partials (d2, index), the screen's partials
// (index, best, second best), the screen's picks and, in the int32 at 16
// bytes before the end, the fp64-pass flag of the last call (1 = it ran)
size_t bank_workspace_bytes(int64_t capacity, int nq) {
  if (bank_small(static_cast<int>(capacity > 1 << 30 ? 1 << 30 : capacity), nq)) return 0;
  const size_t pn = static_cast<size_t>(bank_parts(capacity)) * nq;
  return pn * (sizeof(double) + 2 * sizeof(int64_t) + 2 * sizeof(float)) +
         static_cast<size_t>(nq) * sizeof(int64_t) + 16;
}

cudaError_t launch_bank_check(float* bank, int32_t* count, int32_t* appends, int capacity,
                              int dim, const float* queries, int nq, double thr2, int cap,
                              int32_t* argmin, double* min_d2, uint8_t* appended,
                              DevState* st, int sessions, void* workspace, cudaStream_t s) {
  if (!st && sessions != 1) return cudaErrorInvalidValue;
  if (nq < 1 || nq > kBankMaxQueries) return cudaErrorInvalidValue;
  if (bank_small(capacity, nq)) {
    bank_check_kernel<<<sessions, kBankThreads, 0, s>>>(bank, count, appends, capacity, dim,
                                                        queries, nq, thr2, cap, argmin, min_d2,
                                                        appended, st);
    return cudaGetLastError();
  }
  // large banks: context-free calls only (one session, caller workspace)
  if (st || !workspace) return cudaErrorInvalidValue;
  const size_t smem = sizeof(double) * static_cast<size_t>(nq) * dim;
  const size_t smem32 = smem / 2;
  if (smem > 160 * 1024) return cudaErrorInvalidValue;
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(bank_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return cudaErrorInvalidValue;
  if (smem32 > 48 * 1024 &&
      cudaFuncSetAttribute(bank_screen_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem32)) != cudaSuccess)
    return cudaErrorInvalidValue;
  const int parts = bank_parts(capacity);
  const size_t pn = static_cast<size_t>(parts) * nq;
  double* pd = static_cast<double*>(workspace);
  int64_t* pi = reinterpret_cast<int64_t*>(pd + pn);
  int64_t* si1 = pi + pn;
  int64_t* sel = si1 + pn;
  float* sb1 = reinterpret_cast<float*>(sel + nq);
  float* sb2 = sb1 + pn;
  int32_t* need = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                             bank_workspace_bytes(capacity, nq) - 16);
  // fp32 screen, its decision, the fp64 pass only when a query is undecided,
  // then the in-order decisions (rows the screen does not take: the fp64
  // pass decides alone)
  const bool screen = bank_screen_ok(dim, bank, queries);
  // both passes stride over the entries: persistent grids of as many CTAs as
  // fit on the SMs (fewer partials to merge, a cheap exit for the fp64 pass
  // when it is not needed)
  const int sms = device_sms();
  const int fparts = sms > 0 && parts > 2 * sms ? 2 * sms : parts;
  if (screen) {
    const int sparts = sms > 0 && parts > sms * kScreenBlocks ? sms * kScreenBlocks : parts;
    bank_screen_kernel<<<sparts, kBankThreads, smem32, s>>>(bank, count, capacity, dim, queries, nq,
                                                            sb1, si1, sb2);
    bank_select_kernel<<<1, kBankThreads, 0, s>>>(count, capacity, dim, nq, sb1, si1, sb2, sparts,
                                                  sel, need);
  } else {
    set_flag_kernel<<<1, 1, 0, s>>>(need, 1);
  }
  bank_partial_kernel<<<fparts, kBankThreads, smem, s>>>(bank, count, capacity, dim, queries, nq,
                                                         pd, pi, need);
  bank_resolve_kernel<<<1, kBankThreads, 0, s>>>(bank, count, appends, capacity, dim, queries, nq,
                                                 thr2, cap, pd, pi, fparts, sel, need, argmin,
                                                 min_d2, appended);
  return cudaGetLastError();
}
cudaError_t launch_nearest(const float* store, int count, int dim, const float* query,
                           int32_t* argmin, double* min_d2, cudaStream_t s) {
  nearest_small_kernel<<<1, kBankThreads, 0, s>>>(store, count, dim, query, argmin, min_d2);
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

// Motion cross-attention folded for frame f and head h (32 tokens t, head
// channels d < hd = C / H): with the block's query projection Wq and output
// projection Mo,
//   W_qk[f][c][32 h + t] = fp16(alpha * sum_d Wq[c][hd h + d] K[f][t][hd h + d])
//   VM[f][32 h + t][c]   = fp16(sum_d V[f][t][hd h + d] Mo[hd h + d][c])
// so the block's scores for input rows X are X W_qk[f] (alpha = log2 e /
// sqrt(hd): base-2 logits) and its output is sum_h P_h VM_h = (P V) Mo. Sums
// in fp32, one rounding. Block (h, f, z): rows c of W_qk and columns c of VM
// from 256 z on.
__global__ void __launch_bounds__(256) motion_fold_kernel(const float* __restrict__ kv,
                                                          const __half* __restrict__ wq,
                                                          const __half* __restrict__ mo, int C,
                                                          int H, float alpha, __half* wqk,
                                                          __half* vm) {
  extern __shared__ float skv[];   // K then V of the head: [2][32][hd]
  const int h = blockIdx.x, f = blockIdx.y;
  const int hd = C / H, NT = 32 * H;
  const float* base = kv + static_cast<int64_t>(f) * 32 * 2 * C;
  for (int i = threadIdx.x; i < 32 * hd; i += blockDim.x) {
    const int t = i / hd, d = i - t * hd;
    skv[i] = base[static_cast<int64_t>(t) * 2 * C + h * hd + d];
    skv[32 * hd + i] = base[static_cast<int64_t>(t) * 2 * C + C + h * hd + d];
  }
  __syncthreads();
  const float* sk = skv;
  const float* sv = skv + 32 * hd;
  const int c = blockIdx.z * blockDim.x + threadIdx.x;
  if (c >= C) return;
  // eight head channels at a time: K[t][d0..d0+7] and V[t][..] as two 16-byte
  // broadcast reads each, feeding 8 fmas (hd is a multiple of 8)
  float acc[32];
#pragma unroll
  for (int t = 0; t < 32; ++t) acc[t] = 0.f;
  const __half* wrow = wq + static_cast<int64_t>(c) * C + h * hd;
  for (int d0 = 0; d0 < hd; d0 += 8) {
    float w[8];
    {
      const uint4 u = *reinterpret_cast<const uint4*>(wrow + d0);
      const __half2* hv = reinterpret_cast<const __half2*>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f2 = __half22float2(hv[j]);
        w[2 * j] = f2.x;
        w[2 * j + 1] = f2.y;
      }
    }
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float4 k0 = *reinterpret_cast<const float4*>(sk + t * hd + d0);
      const float4 k1 = *reinterpret_cast<const float4*>(sk + t * hd + d0 + 4);
      float a_ = acc[t];
      a_ = fmaf(w[0], k0.x, a_);
      a_ = fmaf(w[1], k0.y, a_);
      a_ = fmaf(w[2], k0.z, a_);
      a_ = fmaf(w[3], k0.w, a_);
      a_ = fmaf(w[4], k1.x, a_);
      a_ = fmaf(w[5], k1.y, a_);
      a_ = fmaf(w[6], k1.z, a_);
      acc[t] = fmaf(w[7], k1.w, a_);
    }
  }
  __half* o = wqk + (static_cast<int64_t>(f) * C + c) * NT + 32 * h;
#pragma unroll
  for (int t = 0; t < 32; t += 2)
    *reinterpret_cast<__half2*>(o + t) = __floats2half2_rn(alpha * acc[t], alpha * acc[t + 1]);
#pragma unroll
  for (int t = 0; t < 32; ++t) acc[t] = 0.f;
  for (int d0 = 0; d0 < hd; d0 += 8) {
    float m[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) m[j] = __half2float(mo[static_cast<int64_t>(h * hd + d0 + j) * C + c]);
#pragma unroll
    for (int t = 0; t < 32; ++t) {
      const float4 v0 = *reinterpret_cast<const float4*>(sv + t * hd + d0);
      const float4 v1 = *reinterpret_cast<const float4*>(sv + t * hd + d0 + 4);
      float a_ = acc[t];
      a_ = fmaf(v0.x, m[0], a_);
      a_ = fmaf(v0.y, m[1], a_);
      a_ = fmaf(v0.z, m[2], a_);
      a_ = fmaf(v0.w, m[3], a_);
      a_ = fmaf(v1.x, m[4], a_);
      a_ = fmaf(v1.y, m[5], a_);
      a_ = fmaf(v1.z, m[6], a_);
      acc[t] = fmaf(v1.w, m[7], a_);
    }
  }
  __half* v = vm + (static_cast<int64_t>(f) * NT + 32 * h) * C + c;
#pragma unroll
  for (int t = 0; t < 32; ++t) v[static_cast<int64_t>(t) * C] = __float2half_rn(acc[t]);
}

cudaError_t launch_motion_fold(const float* kv, const __half* wq, const __half* mo, int F, int C,
                               int heads, __half* wqk, __half* vm, cudaStream_t s) {
  if (heads < 1 || C % heads || C % 8) return cudaErrorInvalidValue;
  const int hd = C / heads;
  if (hd % 8 || (reinterpret_cast<uintptr_t>(wq) & 15)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * 2 * 32 * hd;
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  const float alpha =
      static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(hd)));
  const dim3 grid(heads, F, (C + 255) / 256);
  motion_fold_kernel<<<grid, 256, smem, s>>>(kv, wq, mo, C, heads, alpha, wqk, vm);
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
