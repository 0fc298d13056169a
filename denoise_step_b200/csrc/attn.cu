// Flash-style attention over KV segments on tcgen05 tensor cores (sm_100a).
//
// One CTA = one (frame, head) pair and two 128-row query tiles. Per KV tile of
// BN keys (segments in order, the concatenation is never materialised):
//   S_i = Q_i K^T                 tcgen05.mma, A and B from shared memory,
//                                 fp32 accumulator in TMEM
//   P_i = exp2(S_i*c - m_i)       softmax warpgroup i: one thread per query
//                                 row, row statistics in fp32, P written back
//                                 to TMEM as fp16 over S_i's columns
//   O_i += P_i V                  tcgen05.mma with A from TMEM (P) and B (V,
//                                 MN-major) from shared memory
// The running maximum is only raised when it grows by more than 2^8, so O is
// rescaled rarely; the final 1/l uses the same maximum as P, so the result is
// the exact softmax up to rounding.
//
// Roles: warp 0 TMA producer (Q once, K/V tiles into a STAGES ring), warp 1
// MMA issuer + TMEM owner, warps 4..7 softmax of query tile 0, warps 8..11
// softmax of query tile 1. The MMA warp interleaves the two tiles so the
// tensor pipe works on one tile while the other one's softmax runs.
#include <cuda_runtime.h>

#include <cmath>

#include "attn.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace pl {

namespace {

template <int HD>
struct Cfg {
  static constexpr int BN = HD > 128 ? 64 : 128;         // keys per tile
  static constexpr int HDP = (HD + 15) / 16 * 16;         // PV MMA N, QK MMA K
  static constexpr int NBLK = (HD + 63) / 64;             // 64-column smem blocks
  static constexpr int KSTEPS = HDP / 16;
  static constexpr int STAGES = NBLK == 1 ? 4 : 2;
  static constexpr uint32_t Q_BLK = 128 * 128;            // one 64-col block of a Q tile
  static constexpr uint32_t Q_BYTES = 2 * NBLK * Q_BLK;
  static constexpr uint32_t KV_BLK = BN * 128;
  static constexpr uint32_t K_BYTES = NBLK * KV_BLK;
  static constexpr uint32_t STAGE_BYTES = 2 * K_BYTES;    // K then V
  static constexpr uint32_t O_COL = 2 * BN;               // TMEM column of O_0
  static constexpr size_t SMEM = Q_BYTES + STAGES * STAGE_BYTES + 1024 + 256;
  static_assert(2 * BN + 2 * HDP <= 512, "TMEM budget");
};

constexpr int kThreads = 384;

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::STAGES * C::STAGE_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_full + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_row0 = blockIdx.x * 256;
  const int head = blockIdx.y;
  const int frame = blockIdx.z;

  int n_active = p.n_total;
  if (p.n_extra != nullptr) {
    int extra = *((volatile const int32_t*)p.n_extra);
    extra = extra < 0 ? 0 : extra;
    const int avail = p.n_total - p.n_fixed;
    n_active = p.n_fixed + (extra < avail ? extra : avail);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_full[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.q);
      mbar_expect_tx(q_full, C::Q_BYTES);
      for (int i = 0; i < 2; ++i)
        for (int b = 0; b < C::NBLK; ++b)
          tma_load_4d(sQ + (i * C::NBLK + b) * C::Q_BLK, &p.q, q_full, 64 * b, head,
                      q_row0 + 128 * i, frame);
      int stage = 0;
      uint32_t phase = 0;
      for (int sg = 0; sg < n_active && !*abort_flag; ++sg) {
        const AttnSeg& seg = p.seg[sg];
        const int fr = seg.per_frame ? frame : 0;
        const int nt = (seg.len + C::BN - 1) / C::BN;
        for (int lt = 0; lt < nt; ++lt) {
          if (!mbar_wait(&kv_empty[stage], phase ^ 1, abort_flag)) break;
          uint8_t* sk = sKV + stage * C::STAGE_BYTES;
          uint8_t* sv = sk + C::K_BYTES;
          mbar_expect_tx(&kv_full[stage], C::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < C::NBLK; ++b)
            tma_load_4d(sk + b * C::KV_BLK, &seg.k, &kv_full[stage], 64 * b, head, lt * C::BN, fr);
#pragma unroll
          for (int b = 0; b < C::NBLK; ++b)
            tma_load_4d(sv + b * C::KV_BLK, &seg.v, &kv_full[stage], 64 * b, head, lt * C::BN, fr);
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, C::HDP, 0, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t kv_base = smem_u32(sKV);
      auto issue_qk = [&](int i, int stage) {
        const uint32_t a0 = q_base + i * C::NBLK * C::Q_BLK;
        const uint32_t b0 = kv_base + stage * C::STAGE_BYTES;
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k) {
          const uint64_t ad = desc_sw128(a0 + (k >> 2) * C::Q_BLK + (k & 3) * 32, 16, 1024);
          const uint64_t bd = desc_sw128(b0 + (k >> 2) * C::KV_BLK + (k & 3) * 32, 16, 1024);
          mma_ss(tmem + i * C::BN, ad, bd, idesc_qk, k > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int i, int stage, bool acc) {
        const uint32_t v0 = kv_base + stage * C::STAGE_BYTES + C::K_BYTES;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k) {
          const uint64_t bd = desc_sw128(v0 + k * 2048, C::KV_BLK, 1024);
          mma_ts(tmem + C::O_COL + i * C::HDP, tmem + i * C::BN + k * 8, bd, idesc_pv,
                 (acc || k > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      int stage = 0, prev_stage = 0;
      uint32_t phase = 0;
      int jt = 0;
      for (int sg = 0; ok && sg < n_active; ++sg) {
        const int nt = (p.seg[sg].len + C::BN - 1) / C::BN;
        for (int lt = 0; lt < nt; ++lt) {
          if (!(ok = mbar_wait(&kv_full[stage], phase, abort_flag))) break;
          tc_fence_after();
          issue_qk(0, stage);
          mma_commit(&s_full[0]);
          if (jt > 0) {
            if (!(ok = mbar_wait(&p_full[1], (jt - 1) & 1, abort_flag))) break;
            tc_fence_after();
            issue_pv(1, prev_stage, jt - 1 > 0);
            mma_commit(&o_full[1]);
            mma_commit(&kv_empty[prev_stage]);
          }
          issue_qk(1, stage);
          mma_commit(&s_full[1]);
          if (!(ok = mbar_wait(&p_full[0], jt & 1, abort_flag))) break;
          tc_fence_after();
          issue_pv(0, stage, jt > 0);
          mma_commit(&o_full[0]);
          prev_stage = stage;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
          ++jt;
        }
      }
      if (ok && jt > 0 && mbar_wait(&p_full[1], (jt - 1) & 1, abort_flag)) {
        tc_fence_after();
        issue_pv(1, prev_stage, jt - 1 > 0);
        mma_commit(&o_full[1]);
        mma_commit(&kv_empty[prev_stage]);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int i = (warp - 4) >> 2;          // query tile of this warpgroup
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int row = 32 * q4 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q4) << 16;
    const uint32_t s_addr = tmem + lane_off + i * C::BN;
    const uint32_t o_addr = tmem + lane_off + C::O_COL + i * C::HDP;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int jt = 0;
    bool ok = true;
    for (int sg = 0; ok && sg < n_active; ++sg) {
      const int len = p.seg[sg].len;
      const int nt = (len + C::BN - 1) / C::BN;
      for (int lt = 0; lt < nt; ++lt) {
        if (!(ok = mbar_wait(&s_full[i], jt & 1, abort_flag))) break;
        tc_fence_after();
        float s[C::BN];
#pragma unroll
        for (int c = 0; c < C::BN; c += 32) tmem_ld32(s_addr + c, reinterpret_cast<uint32_t*>(s + c));
        tmem_wait_ld();
        const int valid = len - lt * C::BN;
        float mx = -INFINITY;
        if (valid < C::BN) {
#pragma unroll
          for (int c = 0; c < C::BN; ++c) {
            s[c] = c < valid ? s[c] : -INFINITY;
            mx = fmaxf(mx, s[c]);
          }
        } else {
#pragma unroll
          for (int c = 0; c < C::BN; ++c) mx = fmaxf(mx, s[c]);
        }
        const float m_tile = mx * sl2;
        const bool need = m_tile > m_run + 8.0f;
        float alpha = 1.0f;
        if (need) {
          alpha = exp2f(m_run - m_tile);
          m_run = m_tile;
        }
        l_run *= alpha;
        if (__any_sync(0xffffffffu, need && jt > 0)) {
          if (!(ok = mbar_wait(&o_full[i], (jt - 1) & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < C::HDP; c0 += 16) {
            uint32_t r[16];
            tmem_ld16(o_addr + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16(o_addr + c0, r);
          }
          tmem_wait_st();
        }
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < C::BN; c += 32) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = exp2f(fmaf(s[c + 2 * e], sl2, -m_run));
            const float p1 = exp2f(fmaf(s[c + 2 * e + 1], sl2, -m_run));
            sum += p0 + p1;
            pk[e] = pack_half2(p0, p1);
          }
          tmem_st16(s_addr + c / 2, pk);
        }
        tmem_wait_st();
        l_run += sum;
        tc_fence_before();
        mbar_arrive(&p_full[i]);
        ++jt;
      }
    }
    if (ok && jt > 0 && mbar_wait(&o_full[i], (jt - 1) & 1, abort_flag)) {
      tc_fence_after();
      const float inv = 1.0f / l_run;
      const int grow = q_row0 + 128 * i + row;
      const bool store = grow < p.n_q;
      __half* orow = p.out + static_cast<int64_t>(frame) * p.out_fstride +
                     static_cast<int64_t>(grow) * p.ldo + static_cast<int64_t>(head) * HD;
#pragma unroll
      for (int c0 = 0; c0 < C::HDP; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(o_addr + c0, r);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            if (c0 + 8 * g < HD) {
              uint4 v;
              v.x = pack_half2(__uint_as_float(r[8 * g + 0]) * inv, __uint_as_float(r[8 * g + 1]) * inv);
              v.y = pack_half2(__uint_as_float(r[8 * g + 2]) * inv, __uint_as_float(r[8 * g + 3]) * inv);
              v.z = pack_half2(__uint_as_float(r[8 * g + 4]) * inv, __uint_as_float(r[8 * g + 5]) * inv);
              v.w = pack_half2(__uint_as_float(r[8 * g + 6]) * inv, __uint_as_float(r[8 * g + 7]) * inv);
              *reinterpret_cast<uint4*>(orow + c0 + 8 * g) = v;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, DEV_TIMEOUT);
}

template <int HD>
int set_attr() {
  return cudaFuncSetAttribute(attn_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(Cfg<HD>::SMEM)) == cudaSuccess ? 0 : 4;
}

template <int HD>
int launch_hd(const AttnParams& p, cudaStream_t stream) {
  using C = Cfg<HD>;
  dim3 grid((p.n_q + 255) / 256, p.heads, p.frames);
  attn_kernel<HD><<<grid, kThreads, C::SMEM, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

}  // namespace

int attn_make_params(AttnParams* p, const void* q, int64_t ldq, int64_t q_fstride,
                     const AttnSegHost* segs, int n_segs, int frames, int n_q, int heads,
                     int head_dim, void* out, int64_t ldo, int64_t out_fstride) {
  if (n_segs < 1 || n_segs > kAttnMaxSegs || frames < 1 || n_q < 1 || heads < 1) return 1;
  if (ldq % 8 || ldo % 8 || q_fstride % 8 || out_fstride % 8) return 1;
  if (ldq < static_cast<int64_t>(heads) * head_dim || ldo < static_cast<int64_t>(heads) * head_dim)
    return 1;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15) return 1;
  const int box_rows_q = 128;
  {
    const int64_t fs = frames > 1 ? q_fstride : static_cast<int64_t>(n_q) * ldq;
    if (frames > 1 && q_fstride <= 0) return 1;
    const uint64_t dims[4] = {static_cast<uint64_t>(head_dim), static_cast<uint64_t>(heads),
                              static_cast<uint64_t>(n_q), static_cast<uint64_t>(frames)};
    const uint64_t strides[3] = {static_cast<uint64_t>(head_dim) * 2,
                                 static_cast<uint64_t>(ldq) * 2, static_cast<uint64_t>(fs) * 2};
    const uint32_t box[4] = {64, 1, static_cast<uint32_t>(box_rows_q), 1};
    if (encode_f16_tmap(&p->q, q, 4, dims, strides, box) != 0) return 2;
  }
  const uint32_t bn = head_dim > 128 ? 64 : 128;
  for (int s = 0; s < n_segs; ++s) {
    const AttnSegHost& h = segs[s];
    if (h.len < 1 || h.len > (1ll << 30) || h.ld % 8 || h.frame_stride % 8 || h.frame_stride < 0)
      return 1;
    if (h.ld < static_cast<int64_t>(heads) * head_dim) return 1;
    if ((reinterpret_cast<uintptr_t>(h.k) | reinterpret_cast<uintptr_t>(h.v)) & 15) return 1;
    const bool per_frame = h.frame_stride != 0 && frames > 1;
    const int64_t fs = per_frame ? h.frame_stride : h.len * h.ld;
    const uint64_t dims[4] = {static_cast<uint64_t>(head_dim), static_cast<uint64_t>(heads),
                              static_cast<uint64_t>(h.len),
                              static_cast<uint64_t>(per_frame ? frames : 1)};
    const uint64_t strides[3] = {static_cast<uint64_t>(head_dim) * 2,
                                 static_cast<uint64_t>(h.ld) * 2, static_cast<uint64_t>(fs) * 2};
    const uint32_t box[4] = {64, 1, bn, 1};
    if (encode_f16_tmap(&p->seg[s].k, h.k, 4, dims, strides, box) != 0) return 2;
    if (encode_f16_tmap(&p->seg[s].v, h.v, 4, dims, strides, box) != 0) return 2;
    p->seg[s].len = static_cast<int>(h.len);
    p->seg[s].per_frame = per_frame ? 1 : 0;
  }
  p->n_fixed = n_segs;
  p->n_total = n_segs;
  p->n_extra = nullptr;
  p->out = static_cast<__half*>(out);
  p->ldo = ldo;
  p->out_fstride = out_fstride;
  p->n_q = n_q;
  p->heads = heads;
  p->frames = frames;
  p->scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  p->status = nullptr;
  return 0;
}

int attn_init() {
  static int done = 0;
  if (!done) {
    if (set_attr<40>() || set_attr<64>() || set_attr<80>() || set_attr<128>() || set_attr<160>())
      return 4;
    done = 1;
  }
  return 0;
}

int attn_launch(const AttnParams& p, int head_dim, cudaStream_t stream) {
  if (attn_init()) return 4;
  switch (head_dim) {
    case 40: return launch_hd<40>(p, stream);
    case 64: return launch_hd<64>(p, stream);
    case 80: return launch_hd<80>(p, stream);
    case 128: return launch_hd<128>(p, stream);
    case 160: return launch_hd<160>(p, stream);
    default: return 7;
  }
}

}  // namespace pl
