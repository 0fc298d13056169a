// Flash-style attention with the PV product transposed, for head_dim <= 64.
//
// At small head dimensions the O = P V product is a stream of thin MMAs
// (M 128 x N 48 x K 16), each costing the tensor pipe about as much as a
// large one. Here each CTA computes O^T = V^T P^T instead: one MMA of
// M 64 (head dims, zero padded) x N 256 (both query tiles) x K 16 covers what
// took two, so a 128-key tile pair needs 6 QK + 8 PV MMAs instead of 22.
//
//   S_i  = Q_i K^T          tcgen05.mma, A/B from shared memory, fp32 in TMEM
//                           (columns 128 i .. 128 i + 127, one buffer per tile)
//   P_i  = exp2(S_i c - m)  softmax warpgroup i, one thread per query row;
//                           the S buffer is released as soon as the row is in
//                           registers, so S(j + 1) overlaps the exps of tile j;
//                           P rows go to shared memory (K-major, 128B swizzle,
//                           two buffers) as the B operand of the PV MMA
//   O^T += V^T P^T          A = the V tile (MN-major), B = P, accumulator
//                           O^T [64 dims x 256 queries] in TMEM columns
//                           256..511 (M = 64 uses lanes 0-15 of each quadrant)
//
// Lazy rescale as in attn.cu: a warpgroup rescales its 128 O^T columns only
// when one of its rows raises its running max by more than 2^8.
#include <cuda_runtime.h>

#include <cmath>

#include "attn.cuh"
#include "fastmath.cuh"
#include "ptx.cuh"

namespace pl {

namespace {

template <int HD>
struct CfgT {
  static constexpr int BN = 128;                         // keys per tile
  static constexpr int HDP = (HD + 15) / 16 * 16;        // QK MMA K (48 at 40, 64 at 64)
  static constexpr int KSTEPS = HDP / 16;
  static constexpr uint32_t Q_TILE = 128 * 128;          // 128 rows x 64 cols fp16
  static constexpr uint32_t Q_BYTES = 2 * Q_TILE;
  static constexpr uint32_t KV_BLK = BN * 128;           // K or V tile: 128 keys x 64 cols
  // K and V have rings of their own: K is released as soon as QK is done, V
  // only after PV, so K of tile j + 2 loads while tile j's softmax runs
  static constexpr int STAGES = 2;
  static constexpr uint32_t P_BLK = 256 * 128;           // 64 keys of P for 256 queries
  static constexpr uint32_t P_BUF = 2 * P_BLK;           // one P buffer (128 keys)
  static constexpr uint32_t P_BYTES = 2 * P_BUF;         // two buffers
  static constexpr uint32_t OT_COL = 256;                // TMEM column of O^T
  static constexpr uint32_t MISC = 2048;                 // barriers, alphas
  static constexpr size_t SMEM = Q_BYTES + 2 * STAGES * KV_BLK + P_BYTES + MISC;
  static_assert(HD <= 64, "transposed PV keeps head dims in one 64-lane M = 64 tile");
  static_assert(SMEM <= 232448, "shared memory budget");
};

constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;      // 384 x 168 >= 128 x 120 + 256 x 184
constexpr int kRegsProducer = 120;
constexpr int kRegsSoftmax = 184;

template <int HD>
__global__ void __launch_bounds__(kThreads, 1) attn_t_kernel(const __grid_constant__ AttnParams p) {
  using C = CfgT<HD>;
  extern __shared__ __align__(1024) uint8_t smem[];
  // The swizzled tiles need 1024-byte alignment and there is no room for
  // slack: refuse to run (status bit) if the base is not aligned.
  if (smem_u32(smem) & 1023) {
    if (threadIdx.x == 0 && p.status) atomicOr(p.status, DEV_BADARG);
    return;
  }
  if (p.box_rows != C::BN) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && p.status)
      atomicOr(p.status, DEV_BADARG);
    return;
  }
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::Q_BYTES;
  uint8_t* sV = sK + C::STAGES * C::KV_BLK;
  uint8_t* sP = sV + C::STAGES * C::KV_BLK;
  uint8_t* misc = sP + C::P_BYTES;
  uint64_t* q_full = reinterpret_cast<uint64_t*>(misc);
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + C::STAGES;
  uint64_t* v_full = k_empty + C::STAGES;
  uint64_t* v_empty = v_full + C::STAGES;
  uint64_t* s_full = v_empty + C::STAGES;    // [2 tiles]: QK done
  uint64_t* s_free = s_full + 2;             // [2 tiles]: row in registers (count 128)
  uint64_t* p_full = s_free + 2;             // [2 buffers]: P of both tiles written (count 256)
  uint64_t* p_free = p_full + 2;             // [2 buffers]: PV done reading the buffer
  uint64_t* o_done = p_free + 2;             // one phase per PV
  uint64_t* o_final = o_done + 1;            // one phase: the last PV done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_final + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* alpha_s = reinterpret_cast<float*>(misc + 1024);   // [256] per-query factors

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
  int nt_total = 0;
  for (int sg = 0; sg < n_active; ++sg) nt_total += (p.seg[sg].len + C::BN - 1) / C::BN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
      mbar_init(&p_full[i], 256);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
  }
  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0 loads Q and the K tiles, warp 2 the V tiles
    if (lane == 0) {
      const bool is_k = warp == 0;
      if (is_k) {
        tma_prefetch_desc(&p.q);
        mbar_expect_tx(q_full, C::Q_BYTES);
        for (int i = 0; i < 2; ++i)
          tma_load_4d(sQ + i * C::Q_TILE, &p.q, q_full, 0, head, q_row0 + 128 * i, frame);
      }
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      uint8_t* ring = is_k ? sK : sV;
      int stage = 0;
      uint32_t phase = 0;
      for (int sg = 0; sg < n_active && !*abort_flag; ++sg) {
        const AttnSeg& seg = p.seg[sg];
        int fr = seg.per_frame ? frame : 0;
        if (seg.block_sel != nullptr) {
          fr = *((volatile const int32_t*)seg.block_sel);
          if (fr < 0 || fr >= seg.n_blocks) {
            if (p.status && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(p.status, DEV_BADARG);
            fr = 0;
          }
        }
        const CUtensorMap* map = is_k ? &seg.k : &seg.v;
        const int nt = (seg.len + C::BN - 1) / C::BN;
        for (int lt = 0; lt < nt; ++lt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
          mbar_expect_tx(&full[stage], C::KV_BLK);
          tma_load_4d(ring + stage * C::KV_BLK, map, &full[stage], 0, head, lt * C::BN, fr);
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
      constexpr uint32_t idesc_pv = idesc_f16_f32(64, 256, 1, 0);   // A = V (MN-major), B = P (K-major)
      const uint64_t dq = desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dv = desc_sw128(smem_u32(sV), C::KV_BLK, 1024);
      const uint64_t dp = desc_sw128(smem_u32(sP), 16, 1024);
      auto issue_qk = [&](int i, int stage) {
        const uint64_t a0 = dq + ((i * C::Q_TILE) >> 4);
        const uint64_t b0 = dk + ((stage * C::KV_BLK) >> 4);
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k)
          mma_ss(tmem + 128 * i, a0 + ((k * 32) >> 4), b0 + ((k * 32) >> 4), idesc_qk,
                 k > 0 ? 1u : 0u);
        mma_commit(&s_full[i]);
      };
      // O^T (+)= V^T(stage) P^T(buffer b), both query tiles at once
      auto issue_pv = [&](int stage, int b, bool acc) {
        const uint64_t a0 = dv + ((stage * C::KV_BLK) >> 4);
        const uint64_t b0 = dp + ((b * C::P_BUF) >> 4);
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          mma_ss(tmem + C::OT_COL, a0 + ((k * 2048) >> 4),
                 b0 + (((k >> 2) * C::P_BLK + (k & 3) * 32) >> 4), idesc_pv,
                 (acc || k > 0) ? 1u : 0u);
        mma_commit(o_done);
        mma_commit(&p_free[b]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag);
      tc_fence_after();
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0;
      auto pv_tile = [&](int t) -> bool {   // PV of tile t (V ring in order)
        const int b = t & 1;
        if (!mbar_wait(&p_full[b], (t >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(&v_full[vs], vph, abort_flag)) return false;
        tc_fence_after();
        issue_pv(vs, b, t > 0);
        mma_commit(&v_empty[vs]);
        if (++vs == C::STAGES) {
          vs = 0;
          vph ^= 1;
        }
        return true;
      };
      int jt = 0;
      for (; ok && jt < nt_total; ++jt) {
        if (!(ok = mbar_wait(&k_full[ks], kph, abort_flag))) break;
        tc_fence_after();
        // S(jt) may overwrite a tile's S buffer once its softmax holds S(jt - 1)
        for (int i = 0; ok && i < 2; ++i) {
          if (jt > 0 && !(ok = mbar_wait(&s_free[i], (jt - 1) & 1, abort_flag))) break;
          tc_fence_after();
          issue_qk(i, ks);
        }
        if (!ok) break;
        mma_commit(&k_empty[ks]);
        if (++ks == C::STAGES) {
          ks = 0;
          kph ^= 1;
        }
        if (jt > 0 && !(ok = pv_tile(jt - 1))) break;
      }
      if (ok && jt > 0 && pv_tile(jt - 1)) mma_commit(o_final);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int i = (warp - 4) >> 2;          // query tile of this warpgroup
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int row = 32 * q4 + lane;         // row in the tile
    const int R = 128 * i + row;            // row in the CTA (P row, O^T column)
    const uint32_t lane_off = static_cast<uint32_t>(32 * q4) << 16;
    const uint32_t s_addr = tmem + lane_off + 128 * i;
    // this warp's O^T lanes: head dims 16 q4 .. 16 q4 + 15 in lanes 0-15 of its quadrant
    const uint32_t ot_addr = tmem + lane_off + C::OT_COL + 128 * i;
    const int bar_id = 1 + i;               // named barrier of this warpgroup
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
        tc_fence_before();
        mbar_arrive(&s_free[i]);
        const int valid = len - lt * C::BN;
        if (valid < C::BN) {
#pragma unroll
          for (int c = 0; c < C::BN; ++c) s[c] = c < valid ? s[c] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mx[a] = s[a];
#pragma unroll
        for (int c = 8; c + 16 <= C::BN; c += 16) {
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = max3f(mx[a], s[c + a], s[c + 8 + a]);
        }
        if constexpr (((C::BN - 8) % 16) != 0) {
#pragma unroll
          for (int a = 0; a < 8; ++a) mx[a] = fmaxf(mx[a], s[C::BN - 8 + a]);
        }
        const float m_tile =
            fmaxf(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], fmaxf(mx[5], fmaxf(mx[6], mx[7])))) * sl2;
        const bool need = m_tile > m_run + 8.0f;
        float alpha = 1.0f;
        if (need) {
          alpha = ex2_f32(m_run - m_tile);
          m_run = m_tile;
        }
        l_run *= alpha;
        if (bar_or(bar_id, 128, need && jt > 0)) {
          // rescale this warpgroup's 128 O^T columns once PV(jt - 1) is in them
          alpha_s[R] = alpha;
          bar_sync(bar_id, 128);
          if (!(ok = mbar_wait(o_done, (jt - 1) & 1, abort_flag))) break;
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(ot_addr + c0, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e)
              r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha_s[128 * i + c0 + e]);
            tmem_st32(ot_addr + c0, r);
          }
          tmem_wait_st();
        }
        // P(jt) goes to buffer jt & 1 once PV(jt - 2) has read it
        const int b = jt & 1;
        if (jt >= 2 && !(ok = mbar_wait(&p_free[b], ((jt >> 1) - 1) & 1, abort_flag))) break;
        const uint64_t sc2 = f2_pack(sl2, sl2);
        const uint64_t nm2 = f2_pack(-m_run, -m_run);
        uint8_t* prow = sP + b * C::P_BUF + (R >> 3) * 1024 + (R & 7) * 128;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < C::BN; c += 32) {
          uint32_t pk[16];
          uint64_t accs[4] = {0, 0, 0, 0};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t x = f2_fma(f2_pack(s[c + 2 * e], s[c + 2 * e + 1]), sc2, nm2);
            float x0, x1;
            f2_unpack(x, x0, x1);
            const uint64_t pp = f2_pack(ex2_f32(x0), ex2_f32(x1));
            accs[e & 3] = f2_add(accs[e & 3], pp);
            float p0, p1;
            f2_unpack(pp, p0, p1);
            pk[e] = h2_from(p0, p1);
          }
          float a0, a1;
          f2_unpack(f2_add(f2_add(accs[0], accs[1]), f2_add(accs[2], accs[3])), a0, a1);
          sum += a0 + a1;
          // keys c .. c + 31 = four 16-byte chunks of the 128B-swizzled row
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = (c >> 3) + q;          // 0..15 over the 128 keys
            uint8_t* dst = prow + (chunk >> 3) * C::P_BLK + (((chunk & 7) ^ (R & 7)) << 4);
            *reinterpret_cast<uint4*>(dst) =
                make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        l_run += sum;
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[b]);
        ++jt;
      }
    }
    if (ok && jt > 0 && mbar_wait(o_final, 0, abort_flag)) {
      tc_fence_after();
      // 1 / l per query column, then each warp writes its 16 head dims of the
      // warpgroup's 128 queries (the first barrier keeps a late rescale's
      // reads of alpha_s ahead of these writes)
      bar_sync(bar_id, 128);
      alpha_s[R] = 1.0f / l_run;
      bar_sync(bar_id, 128);
      const int d = 16 * q4 + lane;            // head dim held by this lane (lanes 0-15)
      const bool dim_ok = lane < 16 && d < HD;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(ot_addr + c0, r);
        tmem_wait_ld();
        if (dim_ok) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int grow = q_row0 + 128 * i + c0 + e;
            if (grow < p.n_q) {
              __half* o = p.out + static_cast<int64_t>(frame) * p.out_fstride +
                          static_cast<int64_t>(grow) * p.ldo + static_cast<int64_t>(head) * HD + d;
              *o = __float2half_rn(__uint_as_float(r[e]) * alpha_s[128 * i + c0 + e]);
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
int set_attr_t() {
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, attn_t_kernel<HD>) != cudaSuccess) return 4;
  if (fa.numRegs != kRegsLaunch) return 4;
  return cudaFuncSetAttribute(attn_t_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(CfgT<HD>::SMEM)) == cudaSuccess ? 0 : 4;
}

}  // namespace

int attn_t_block_n() { return CfgT<64>::BN; }

int attn_t_init() {
  static int done = 0;
  if (!done) {
    if (set_attr_t<40>() || set_attr_t<64>()) return 4;
    done = 1;
  }
  return 0;
}

int attn_t_launch(const AttnParams& p, int head_dim, cudaStream_t stream) {
  if (attn_t_init()) return 4;
  dim3 grid((p.n_q + 255) / 256, p.heads, p.frames);
  switch (head_dim) {
    case 40: attn_t_kernel<40><<<grid, kThreads, CfgT<40>::SMEM, stream>>>(p); break;
    case 64: attn_t_kernel<64><<<grid, kThreads, CfgT<64>::SMEM, stream>>>(p); break;
    default: return 7;
  }
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

}  // namespace pl
