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
// the exact softmax up to rounding. Where head_dim sits below its 16-column
// padding (40 -> 48) the row sum l comes from the tensor core: V's first
// padding column is set to 1 in shared memory (warp 3, after each K/V tile
// lands), so PV accumulates l = sum_k P[:, k] into O[:, head_dim], in the
// same fp16 P as the numerator and rescaled with it (level-64 launch 3.11 ->
// 2.95 ms: 48 packed adds per softmax warp and tile fewer).
//
// Roles: warpgroup 0 = warp 0 TMA producer (Q once, K/V tiles into a STAGES
// ring), warp 1 MMA issuer of query tile 0 and TMEM owner, warp 2 MMA issuer
// of query tile 1 when each tile has two S buffers (else warp 1 issues both,
// which measured faster there); warp 3 writes V's ones column where the row
// sums come from the tensor core (else idle); warpgroups 1 and 2 = softmax of
// query tiles 0 and 1.
// setmaxnreg moves registers from warpgroup 0 (120 per thread) to the softmax
// warpgroups (184 per thread); the launch is refused unless the kernel was
// compiled at 168 registers per thread, the exact total that split needs.
//
// The softmax is issue- and MUFU-bound (one exp2 per score at head_dim 40
// against 160 tensor FLOPs), so its inner loop uses packed f32x2 FMAs,
// 3-input max and one of two exp2 paths (EXPM): 0 = ex2.approx.f32 on the
// MUFU pipe; 2 = MUFU for most pairs and a degree-3 polynomial on the FMA
// pipe for the pairs kPolyPairs marks (Cody-Waite split 2^x = 2^n 2^f with n
// the nearest integer, f in [-0.5, 0.5]; the cubic is fitted to 2^f on that
// interval, max relative error 7.7e-5, below the fp16 rounding of P).
// Measured on B200 (level-64 kernel): ex2.approx.f32 issues 16 results per
// clock per SM and ex2.approx.f16x2 only 8 instructions (the same 16 results),
// so the f16x2 path was dropped. With one MMA issuer the polynomial split was
// slower (the tensor pipe set the pace); with two it takes 8% off head_dim 40.
#include <cuda_runtime.h>

#include <cmath>
#include <mutex>

#include "attn.cuh"
#include "devinit.cuh"
#include "fastmath.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace pl {

namespace {

template <int HD, int VAR = 0>
struct Cfg {
  // VAR 0: 128-key tiles, one S buffer per query tile (64 keys at head_dim 160);
  // VAR 1: 64-key tiles, two S buffers per query tile where TMEM allows;
  // VAR 2: 96-key tiles with two S buffers where they fit (head_dim <= 64),
  //        else as VAR 0
  static constexpr bool V2 = VAR == 2 && 4 * 96 + 2 * ((HD + 15) / 16 * 16) <= 512;
  static constexpr int BN = V2 ? 96 : ((VAR == 1 || HD > 128) ? 64 : 128);  // keys per tile
  static constexpr int HDP = (HD + 15) / 16 * 16;         // PV MMA N, QK MMA K
  static constexpr int NBLK = (HD + 63) / 64;             // 64-column smem blocks
  static constexpr int KSTEPS = HDP / 16;
  // S buffers per query tile: 2 (S of the next KV tile is computed while the
  // softmax works on this one) when 4 S buffers and 2 O accumulators fit in
  // the 512 TMEM columns, else 1
  static constexpr int SB = ((VAR == 1 || V2) && 4 * BN + 2 * HDP <= 512) ? 2 : 1;
  static constexpr uint32_t Q_BLK = 128 * 128;            // one 64-col block of a Q tile
  static constexpr uint32_t Q_BYTES = 2 * NBLK * Q_BLK;
  static constexpr uint32_t KV_BLK = BN * 128;
  static constexpr uint32_t K_BYTES = NBLK * KV_BLK;
  static constexpr uint32_t STAGE_BYTES = 2 * K_BYTES;    // K then V
  static constexpr int STAGES = (NBLK == 1 ? 8 : (NBLK == 2 ? 4 : 2)) * 64 / BN;
  static_assert(BN % 32 == 0 && STAGES >= 2, "tile shape");
  static constexpr uint32_t O_COL = 2 * SB * BN;          // TMEM column of O_0
  static constexpr size_t SMEM = Q_BYTES + STAGES * STAGE_BYTES + 1024 + 512;
  // head_dim below its 16-column padding: V's first padding column is set to
  // 1 in shared memory, so PV also accumulates the row sum l of P into
  // O[:, HD] (the softmax keeps no sums)
  static constexpr bool ONES = HDP > HD;
  static_assert(2 * SB * BN + 2 * HDP <= 512, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  // barriers, TMEM slot, abort flag and segment lengths fit the 512-byte tail
  static_assert(8 * (20 + 3 * STAGES + 2 * SB) + 8 + 4 * kAttnMaxSegs <= 512, "barrier area");
};

constexpr int kThreads = 384;
// EXPM 2: bit e set = pair e of each 32-column chunk takes the FMA-pipe exp2
constexpr uint32_t kPolyPairs = 0x9248u;
constexpr int kRegsLaunch = 168;      // 384 x 168 >= 128 x 120 + 256 x 184
constexpr int kRegsProducer = 120;
constexpr int kRegsSoftmax = 184;

template <int HD, int EXPM, int VAR>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const __grid_constant__ AttnParams p) {
  using C = Cfg<HD, VAR>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + C::STAGES * C::STAGE_BYTES);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + C::STAGES;
  uint64_t* s_full = kv_empty + C::STAGES;   // [2 tiles][SB]
  uint64_t* p_full = s_full + 2 * C::SB;     // [2 tiles][2]
  uint64_t* o_full = p_full + 4;             // [2 tiles]: one phase per PV (one S buffer) or
                                             // one phase for the next-to-last PV (two S buffers)
  uint64_t* o_final = o_full + 2;            // [2 tiles], one phase: the tile's last PV done
  uint64_t* stagger = o_final + 2;           // one phase: tile 0 has reached its first exps
  uint64_t* v_ready = stagger + 1;           // [STAGES]: V's ones column written (ONES)
  uint64_t* drain = v_ready + C::STAGES;     // [2 issuers]: their MMAs done (after an abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  // segment lengths, copied once from the parameter space (a constant-cache
  // miss costs several hundred clocks on a warp's critical path)
  int* seg_len = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q_row0 = blockIdx.x * 256;
  const int head = blockIdx.y;
  const int frame = blockIdx.z;
  const uint64_t wl = p.wait_ns;   // limit of every bounded wait

  // the K/V boxes the host encoded must match this kernel's key tile, or the
  // TMA writes would not fit the stage buffers: refuse to run
  if (p.box_rows != C::BN) {
    if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && p.status)
      atomicOr(p.status, DEV_BADARG);
    return;
  }

  int n_active = p.n_total;
  if (p.n_extra != nullptr) {
    const int si = p.extra_div > 0 ? frame / p.extra_div : 0;
    int extra = *((volatile const int32_t*)(p.n_extra + static_cast<int64_t>(si) * p.extra_stride));
    extra = extra < 0 ? 0 : extra;
    const int avail = p.n_total - p.n_fixed;
    n_active = p.n_fixed + (extra < avail ? extra : avail);
  }

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], C::SB == 2 ? 2 : 1);   // one commit per MMA issuer
    }
    for (int b = 0; b < 2 * C::SB; ++b) mbar_init(&s_full[b], 1);
    for (int b = 0; b < 4; ++b) mbar_init(&p_full[b], 128);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&o_full[i], 1);
      mbar_init(&o_final[i], 1);
    }
    mbar_init(stagger, 128);
    for (int s = 0; s < C::STAGES; ++s) mbar_init(&v_ready[s], 1);
    for (int w = 0; w < 2; ++w) mbar_init(&drain[w], 1);
    for (int sg = 0; sg < n_active; ++sg) seg_len[sg] = p.seg[sg].len;
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // TMEM column of S buffer b of query tile i, and of O_i
  auto s_col = [](int i, int b) { return static_cast<uint32_t>((i * C::SB + b) * C::BN); };
  auto o_col = [](int i) { return static_cast<uint32_t>(C::O_COL + i * C::HDP); };

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
  }
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
      int issued = 0;   // K/V tiles whose copies were started
      // planted failure (test hook): no K/V tile is loaded, so the consumers'
      // bounded waits run out with no copy in flight
      const int n_load = p.test_mode == kTestNoKV ? 0 : n_active;
      for (int sg = 0; sg < n_load && !*abort_flag; ++sg) {
        const AttnSeg& seg = p.seg[sg];
        int fr = seg.per_frame ? frame : (seg.frame_div > 0 ? frame / seg.frame_div : 0);
        if (seg.block_sel != nullptr) {
          fr = *((volatile const int32_t*)seg.block_sel);
          if (fr < 0 || fr >= seg.n_blocks) {   // out of range: attend block 0, flag it
            if (p.status && blockIdx.x == 0 && blockIdx.y == 0) atomicOr(p.status, DEV_BADARG);
            fr = 0;
          }
        }
        const int nt = (seg.len + C::BN - 1) / C::BN;
        for (int lt = 0; lt < nt; ++lt) {
          if (!mbar_wait(&kv_empty[stage], phase ^ 1, abort_flag, wl)) break;
          uint8_t* sk = sKV + stage * C::STAGE_BYTES;
          uint8_t* sv = sk + C::K_BYTES;
          mbar_expect_tx(&kv_full[stage], C::STAGE_BYTES);
#pragma unroll
          for (int b = 0; b < C::NBLK; ++b)
            tma_load_4d(sk + b * C::KV_BLK, &seg.k, &kv_full[stage], 64 * b, head, lt * C::BN, fr);
#pragma unroll
          for (int b = 0; b < C::NBLK; ++b)
            tma_load_4d(sv + b * C::KV_BLK, &seg.v, &kv_full[stage], 64 * b, head, lt * C::BN, fr);
          ++issued;
          if (++stage == C::STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // let the copies still in flight (at most the last STAGES tiles and
        // Q) land before the CTA's shared memory can go to another CTA
        mbar_wait_drain(q_full, 0, wl);
        for (int t = issued > C::STAGES ? issued - C::STAGES : 0; t < issued; ++t)
          mbar_wait_drain(&kv_full[t % C::STAGES], (t / C::STAGES) & 1, wl);
      }
    }
    __syncwarp();
  } else if (warp == 1 || (C::SB == 2 && warp == 2)) {
    // ------------------------------------------------------------ MMA issuer(s)
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, C::BN, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16_f32(128, C::HDP, 0, 1);
      // Descriptor templates: the start-address field (bits 0-13) holds
      // address >> 4, so adding (byte offset >> 4) moves a descriptor inside
      // shared memory; all offsets below are compile-time except the stage.
      const uint64_t dq = desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dk = desc_sw128(smem_u32(sKV), 16, 1024);
      const uint64_t dv = desc_sw128(smem_u32(sKV) + C::K_BYTES, C::KV_BLK, 1024);
      auto issue_qk = [&](int i, int stage, int b) {
        const uint64_t a0 = dq + ((i * C::NBLK * C::Q_BLK) >> 4);
        const uint64_t b0 = dk + ((stage * C::STAGE_BYTES) >> 4);
        const uint32_t d = tmem + s_col(i, b);
#pragma unroll
        for (int k = 0; k < C::KSTEPS; ++k) {
          const uint32_t off = ((k >> 2) * C::Q_BLK + (k & 3) * 32) >> 4;
          const uint32_t offk = ((k >> 2) * C::KV_BLK + (k & 3) * 32) >> 4;
          mma_ss(d, a0 + off, b0 + offk, idesc_qk, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[i * C::SB + b]);
      };
      // O_i (+)= P_i V with P read from S buffer b (fp16, two keys per column)
      auto issue_pv = [&](int i, int stage, int b, bool acc, bool commit_o = true) {
        const uint64_t v0 = dv + ((stage * C::STAGE_BYTES) >> 4);
        const uint32_t d = tmem + o_col(i);
        const uint32_t a = tmem + s_col(i, b);
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          mma_ts(d, a + k * 8, v0 + ((k * 2048) >> 4), idesc_pv, (acc || k > 0) ? 1u : 0u);
        if (commit_o) mma_commit(&o_full[i]);
      };
      auto wait_p = [&](int i, int jt) {
        const bool r = mbar_wait(&p_full[i * 2 + (jt & 1)], (jt >> 1) & 1, abort_flag, wl);
        tc_fence_after();
        return r;
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, wl);
      tc_fence_after();
      // the MMA side only needs the total tile count (the tiles' segments
      // matter to the producer and the softmax)
      int nt_total = 0;
      for (int sg = 0; sg < n_active; ++sg) nt_total += (seg_len[sg] + C::BN - 1) / C::BN;
      int stage = 0;
      uint32_t phase = 0;
      auto next_stage = [&]() {
        if (++stage == C::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      };
      if constexpr (C::SB == 2) {
        // Two issuers: warp 1 runs query tile 0's MMAs and warp 2 tile 1's.
        // A shared-memory access by an issuing thread (an mbarrier wait
        // included) is ordered behind the MMAs it has queued, so each wait
        // lets that thread's queue run dry; with two independent issuers the
        // tensor pipe executes one tile's MMAs while the other's issuer waits
        // (measured on B200: 18 MMAs of this shape per KV tile in ~1100
        // clocks with two issuers against ~1900 with one).
        // Each tile's S runs two KV tiles ahead of its PV: PV_i(j) frees the
        // S buffer that QK_i(j + 2) fills. PV completion needs no commit of
        // its own: S_i(j + 2) landing implies PV_i(j) has (one issuer, in-order
        // pipe), which is what the softmax waits on before a rescale; only the
        // next-to-last PV, which no QK follows, commits o_full. A K/V stage is
        // released by both issuers' commits.
        static_assert(C::STAGES >= 3, "three KV tiles are in flight");
        const int i = warp - 1;
        auto stage_of = [](int t) { return t % C::STAGES; };
        auto wait_kv = [&](int t) {
          const bool r = mbar_wait(&kv_full[stage_of(t)], (t / C::STAGES) & 1, abort_flag, wl);
          tc_fence_after();
          return r;
        };
        for (int t = 0; ok && t < 2 && t < nt_total; ++t) {
          if (!(ok = wait_kv(t))) break;
          issue_qk(i, stage_of(t), t);
        }
        for (int jt = 0; ok && jt < nt_total; ++jt) {
          const int st = stage_of(jt);
          const int b = jt & 1;
          const bool ahead = jt + 2 < nt_total;
          if (!(ok = wait_p(i, jt))) break;
          if (ahead && !(ok = wait_kv(jt + 2))) break;
          if (C::ONES) {
            if (!(ok = mbar_wait(&v_ready[st], (jt / C::STAGES) & 1, abort_flag, wl))) break;
            tc_fence_after();
          }
          issue_pv(i, st, b, jt > 0, jt == nt_total - 2);
          if (jt == nt_total - 1) mma_commit(&o_final[i]);
          mma_commit(&kv_empty[st]);
          if (ahead) issue_qk(i, stage_of(jt + 2), b);
        }
      } else {
        int prev_stage = 0;
        int jt = 0;
        for (; ok && jt < nt_total; ++jt) {
          if (!(ok = mbar_wait(&kv_full[stage], phase, abort_flag, wl))) break;
          tc_fence_after();
          // one S buffer per tile: PV(jt - 1) must be issued before S(jt)
          // overwrites the P it reads (the tensor pipe runs them in order)
          issue_qk(0, stage, 0);
          if (jt > 0) {
            if (!(ok = wait_p(1, jt - 1))) break;
            issue_pv(1, prev_stage, 0, jt - 1 > 0);
            mma_commit(&kv_empty[prev_stage]);
          }
          issue_qk(1, stage, 0);
          if (!(ok = wait_p(0, jt))) break;
          issue_pv(0, stage, 0, jt > 0);
          prev_stage = stage;
          next_stage();
        }
        if (ok && jt > 0) {
          // tile 0's last PV was issued inside the loop
          mma_commit(&o_final[0]);
          if (wait_p(1, jt - 1)) {
            issue_pv(1, prev_stage, 0, jt - 1 > 0);
            mma_commit(&o_final[1]);
            mma_commit(&kv_empty[prev_stage]);
          }
        }
      }
      if (*abort_flag) {
        // the MMAs this thread queued must finish before TMEM is freed
        mma_commit(&drain[warp - 1]);
        mbar_wait_drain(&drain[warp - 1], 0, wl);
      }
    }
    __syncwarp();
  } else if (C::ONES && warp == 3) {
    // ------------------------------------------------------------ ones column
    // V[:, HD] := 1 in each K/V stage once its tile has landed (the TMA
    // zero-fills the padding columns); 128-byte swizzle: 16-byte unit u of
    // row r sits at unit u ^ (r & 7)
    int nt_total = 0;
    for (int sg = 0; sg < n_active; ++sg) nt_total += (seg_len[sg] + C::BN - 1) / C::BN;
    constexpr uint32_t kBlk = HD / 64, kUnit = (HD % 64) * 2 / 16, kByte = (HD % 64) * 2 % 16;
    for (int t = 0; t < nt_total; ++t) {
      const int st = t % C::STAGES;
      if (!mbar_wait(&kv_full[st], (t / C::STAGES) & 1, abort_flag, wl)) break;
      uint8_t* sv = sKV + st * C::STAGE_BYTES + C::K_BYTES + kBlk * C::KV_BLK;
      for (int r = lane; r < C::BN; r += 32)
        *reinterpret_cast<__half*>(sv + r * 128 + (((kUnit ^ (r & 7)) << 4) | kByte)) =
            __float2half(1.0f);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_ready[st]);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    const int i = (warp - 4) >> 2;          // query tile of this warpgroup
    const int q4 = warp & 3;                // TMEM lane quadrant
    const int row = 32 * q4 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q4) << 16;
    const uint32_t o_addr = tmem + lane_off + o_col(i);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    int jt = 0;
    bool ok = true;
    // With two S buffers the two tiles' S supplies are independent, so
    // warpgroup 1 starts its first tile only when warpgroup 0 begins its
    // first exps: the warpgroups' exp phases then start out of step and
    // interleave on the MUFU for the first KV tiles instead of coinciding
    // (measured 3% faster over a level-64 launch; in steady state the two
    // drift back into step). Only on the 96-key schedule: with 64-key tiles
    // (head_dim 80) it measured 1.3% slower and with 96-key ones without it
    // 1% slower.
    int nt_all = 0;
    for (int sg = 0; sg < n_active; ++sg) nt_all += (seg_len[sg] + C::BN - 1) / C::BN;
    if (C::V2 && C::SB == 2 && i == 1 && n_active > 0) ok = mbar_wait(stagger, 0, abort_flag, wl);
    for (int sg = 0; ok && sg < n_active; ++sg) {
      const int len = seg_len[sg];
      const int nt = (len + C::BN - 1) / C::BN;
      for (int lt = 0; lt < nt; ++lt) {
        const int b = C::SB == 2 ? (jt & 1) : 0;
        const uint32_t use = C::SB == 2 ? static_cast<uint32_t>(jt >> 1) : static_cast<uint32_t>(jt);
        if (!(ok = mbar_wait(&s_full[i * C::SB + b], use & 1, abort_flag, wl))) break;
        tc_fence_after();
        const uint32_t s_addr = tmem + lane_off + s_col(i, b);
        float s[C::BN];
#pragma unroll
        for (int c = 0; c < C::BN; c += 32) tmem_ld32(s_addr + c, reinterpret_cast<uint32_t*>(s + c));
        tmem_wait_ld();
        const int valid = len - lt * C::BN;
        if (valid < C::BN) {
#pragma unroll
          for (int c = 0; c < C::BN; ++c) s[c] = c < valid ? s[c] : -INFINITY;
        }
        // row max as 8 independent max3 chains (short dependency depth)
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
        const float m_tile = fmaxf(max3f(mx[0], mx[1], mx[2]), max3f(mx[3], mx[4], fmaxf(mx[5], fmaxf(mx[6], mx[7])))) * sl2;
        const bool need = m_tile > m_run + 8.0f;
        float alpha = 1.0f;
        if (need) {
          alpha = ex2_f32(m_run - m_tile);
          m_run = m_tile;
        }
        l_run *= alpha;
        if (__any_sync(0xffffffffu, need && jt > 0)) {
          // rescale O_i once PV(jt - 1) has landed in it: with two S buffers
          // S_i(jt + 1) is issued after PV_i(jt - 1), so its barrier serves
          // (the softmax waits on that phase next anyway); PV(nt - 2) has its
          // own one-shot phase on o_full
          if constexpr (C::SB == 2) {
            const bool via_s = jt + 1 < nt_all;
            ok = via_s ? mbar_wait(&s_full[i * C::SB + ((jt + 1) & 1)], ((jt + 1) >> 1) & 1, abort_flag, wl)
                       : mbar_wait(&o_full[i], 0, abort_flag, wl);
          } else {
            ok = mbar_wait(&o_full[i], (jt - 1) & 1, abort_flag, wl);
          }
          if (!ok) break;
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
        if (C::SB == 2 && i == 0 && jt == 0) mbar_arrive(stagger);
        const uint64_t sc2 = f2_pack(sl2, sl2);
        const uint64_t nm2 = f2_pack(-m_run, -m_run);
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < C::BN; c += 32) {
          uint32_t pk[16];
          {
            uint64_t accs[4] = {0, 0, 0, 0};
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const uint64_t x = f2_fma(f2_pack(s[c + 2 * e], s[c + 2 * e + 1]), sc2, nm2);
              uint64_t pp;
              if (EXPM == 2 && ((kPolyPairs >> e) & 1)) {
                pp = exp2_poly2(x);
              } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                pp = f2_pack(ex2_f32(x0), ex2_f32(x1));
              }
              if constexpr (!C::ONES) accs[e & 3] = f2_add(accs[e & 3], pp);
              float p0, p1;
              f2_unpack(pp, p0, p1);
              pk[e] = h2_from(p0, p1);
            }
            if constexpr (!C::ONES) {
              float a0, a1;
              f2_unpack(f2_add(f2_add(accs[0], accs[1]), f2_add(accs[2], accs[3])), a0, a1);
              sum += a0 + a1;
            }
          }
          tmem_st16(s_addr + c / 2, pk);
        }
        tmem_wait_st();
        l_run += sum;
        tc_fence_before();
        mbar_arrive(&p_full[i * 2 + (jt & 1)]);
        ++jt;
      }
    }
    // o_final has a single phase, so this wait cannot be satisfied by an
    // earlier PV (with two S buffers the last two PVs can both be in flight)
    if (ok && jt > 0 && mbar_wait(&o_final[i], 0, abort_flag, wl)) {
      tc_fence_after();
      float l_fin = l_run;
      if constexpr (C::ONES) {
        uint32_t r[16];
        tmem_ld16(o_addr + HD / 16 * 16, r);
        tmem_wait_ld();
        l_fin = __uint_as_float(r[HD % 16]);
      }
      const float inv = 1.0f / l_fin;
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

// Tile schedule per head dimension (measured on B200 with the two MMA
// issuers): 96-key tiles with two S buffers per query tile where TMEM holds
// them (head_dim <= 64), 64-key tiles with two S buffers up to head_dim 128
// (level-32 layer 0.355 -> 0.303 ms against 128-key single-buffered tiles,
// PR-Sink block 2.02 -> 1.94 ms), 64-key single-buffered tiles with one
// issuer at head_dim 160.
template <int HD>
constexpr int kVar = (HD <= 64) ? 2 : (HD <= 128 ? 1 : 0);
// exp2 path per head dimension: at head_dim <= 64 the MUFU is the limit and
// 5 of every 16 pairs go to the FMA-pipe polynomial (level-64 launch 3.39 ->
// 3.12 ms; 4/16: 3.20, 6/16: 3.28, 2/16: 3.36 ms); at larger head dims the
// tensor pipe leads and the polynomial measured slower (32x32 layer 0.307 ->
// 0.317 ms, PR-Sink block 1.91 -> 2.00 ms), so MUFU only there.
template <int HD>
constexpr int kExpMode = (HD <= 64) ? 2 : 0;

int block_n(int head_dim) {
  switch (head_dim) {
    case 40: return Cfg<40, kVar<40>>::BN;
    case 64: return Cfg<64, kVar<64>>::BN;
    case 80: return Cfg<80, kVar<80>>::BN;
    case 128: return Cfg<128, kVar<128>>::BN;
    case 160: return Cfg<160, kVar<160>>::BN;
    default: return 0;
  }
}

template <int HD>
int set_attr() {
  constexpr int V = kVar<HD>;
  // the setmaxnreg split needs exactly kRegsLaunch registers per thread at launch
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, attn_kernel<HD, kExpMode<HD>, V>) != cudaSuccess) return 4;
  if (fa.numRegs != kRegsLaunch) return 4;
  return cudaFuncSetAttribute(attn_kernel<HD, kExpMode<HD>, V>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(Cfg<HD, V>::SMEM)) == cudaSuccess ? 0 : 4;
}

template <int HD>
int launch_hd(const AttnParams& p, cudaStream_t stream) {
  constexpr int V = kVar<HD>;
  dim3 grid((p.n_q + 255) / 256, p.heads, p.frames);
  attn_kernel<HD, kExpMode<HD>, V><<<grid, kThreads, Cfg<HD, V>::SMEM, stream>>>(p);
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
  const int bn_i = block_n(head_dim);
  if (bn_i == 0) return 7;
  const uint32_t bn = static_cast<uint32_t>(bn_i);
  for (int s = 0; s < n_segs; ++s) {
    const AttnSegHost& h = segs[s];
    if (h.len < 1 || h.len > (1ll << 30) || h.ld % 8 || h.frame_stride % 8 || h.frame_stride < 0)
      return 1;
    if (h.ld < static_cast<int64_t>(heads) * head_dim) return 1;
    if ((reinterpret_cast<uintptr_t>(h.k) | reinterpret_cast<uintptr_t>(h.v)) & 15) return 1;
    const bool stacked = h.block_sel != nullptr || h.frame_div > 0;
    if (h.block_sel != nullptr && h.frame_div > 0) return 1;
    if (h.frame_div < 0) return 1;
    if (stacked && (h.n_blocks < 1 || h.frame_stride <= 0)) return 1;
    // every frame's block must exist
    if (h.frame_div > 0 && (frames - 1) / h.frame_div >= h.n_blocks) return 1;
    const bool per_frame = !stacked && h.frame_stride != 0 && frames > 1;
    const int64_t fs = (per_frame || stacked) ? h.frame_stride : h.len * h.ld;
    const uint64_t n4 = stacked ? static_cast<uint64_t>(h.n_blocks) : (per_frame ? frames : 1);
    const uint64_t dims[4] = {static_cast<uint64_t>(head_dim), static_cast<uint64_t>(heads),
                              static_cast<uint64_t>(h.len), n4};
    const uint64_t strides[3] = {static_cast<uint64_t>(head_dim) * 2,
                                 static_cast<uint64_t>(h.ld) * 2, static_cast<uint64_t>(fs) * 2};
    const uint32_t box[4] = {64, 1, bn, 1};
    if (encode_f16_tmap(&p->seg[s].k, h.k, 4, dims, strides, box) != 0) return 2;
    if (encode_f16_tmap(&p->seg[s].v, h.v, 4, dims, strides, box) != 0) return 2;
    p->seg[s].len = static_cast<int>(h.len);
    p->seg[s].per_frame = per_frame ? 1 : 0;
    p->seg[s].block_sel = h.block_sel;
    p->seg[s].n_blocks = static_cast<int>(n4);
    p->seg[s].frame_div = h.frame_div;
  }
  p->n_fixed = n_segs;
  p->n_total = n_segs;
  p->n_extra = nullptr;
  p->extra_div = 0;
  p->extra_stride = 0;
  p->out = static_cast<__half*>(out);
  p->ldo = ldo;
  p->out_fstride = out_fstride;
  p->n_q = n_q;
  p->heads = heads;
  p->frames = frames;
  p->scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  p->box_rows = bn_i;
  p->status = nullptr;
  p->wait_ns = kWaitLimitNs;
  p->test_mode = 0;
  return 0;
}

int attn_init() {
  // kernel attributes are per device: set them once on each device used
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return 4;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (set_attr<40>() || set_attr<64>() || set_attr<80>() || set_attr<128>() || set_attr<160>())
      return 4;
    done[dev] = true;
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
