// Persistent, warp-specialised fp16 GEMM on tcgen05 tensor cores.
//
//   warp 0      TMA producer: A tile [128 x 64] (K-major) + B tile [64 x BN]
//               (MN-major, BN/64 column blocks), 128-byte swizzle, STAGES ring
//   warp 1      MMA issuer (one lane): 4 x tcgen05.mma (K = 16) per stage into
//               a TMEM accumulator; two accumulators alternate between tiles.
//               It waits for two stages at a time: a wait by the issuing
//               thread is ordered behind the MMAs it has queued, so each one
//               lets the tensor pipe run dry for a moment.
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (one TMEM lane = one
//               row, 32 columns at a time), fp32 -> fp16 (or kept fp32) into a
//               swizzled shared-memory chunk of 32 rows x 32 columns, written
//               out by a TMA tile store (two chunks in flight per warp)
#include <cuda_runtime.h>

#include <mutex>

#include "devinit.cuh"
#include "gemm.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace pl {

namespace {

constexpr int kStages = 4;
constexpr int kNB = (kGemmBN + 63) / 64;            // 64-column B blocks per tile
constexpr uint32_t kABytes = kGemmBM * 128;          // 128 rows x 128 B
constexpr uint32_t kBBlockBytes = 64 * 128;          // 64 K-rows x 128 B
constexpr uint32_t kBBytes = kNB * kBBlockBytes;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kAccStride = 256;                 // TMEM columns per accumulator
constexpr int kThreads = 192;
constexpr uint32_t kChunkBytes = 32 * 128;           // 32 rows x 32 columns, fp32 worst case
constexpr uint32_t kStagingBytes = 4 * 2 * kChunkBytes;   // 4 epilogue warps x 2 chunks
constexpr size_t kSmemBytes = kStages * kStageBytes + kStagingBytes + 1024 + 256;
static_assert(kGemmBN % 32 == 0, "32-column epilogue chunks");

struct TileCoord {
  int prob, m0, n0;
};

__device__ __forceinline__ bool decode_tile(const GemmParams& p, int t, TileCoord& tc) {
  int pi = 0;
  while (pi < p.n_problems - 1 && t >= p.prob[pi].tile_end) ++pi;
  const GemmProblem& pr = p.prob[pi];
  if (pr.pred != nullptr && *((volatile const int32_t*)pr.pred) == 0) return false;
  const int local = t - pr.tile_begin;
  tc.prob = pi;
  tc.m0 = (local / pr.tiles_n) * kGemmBM;
  tc.n0 = (local % pr.tiles_n) * kGemmBN;
  return true;
}

__global__ void __launch_bounds__(kThreads, 1) gemm_f16_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* staging = smem + kStages * kStageBytes;     // 1024-byte aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kStagingBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;      // the issuer's MMAs done (after an abort)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < p.n_problems; ++i) {
        tma_prefetch_desc(&p.prob[i].a);
        tma_prefetch_desc(&p.prob[i].b);
      }
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;   // stages whose copies were started
      for (int t = blockIdx.x; t < p.total_tiles && !*abort_flag; t += gridDim.x) {
        TileCoord tc;
        if (!decode_tile(p, t, tc)) continue;
        const GemmProblem& pr = p.prob[tc.prob];
        const int nk = (pr.K + kGemmBK - 1) / kGemmBK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) break;
          ++issued;
          uint8_t* sa = smem + stage * kStageBytes;
          uint8_t* sb = sa + kABytes;
          mbar_expect_tx(&full[stage], kStageBytes);
          tma_load_2d(sa, &pr.a, &full[stage], kb * kGemmBK, tc.m0);
#pragma unroll
          for (int j = 0; j < kNB; ++j)
            tma_load_2d(sb + j * kBBlockBytes, &pr.b, &full[stage], tc.n0 + 64 * j, kb * kGemmBK);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) {
        // let the copies still in flight land before the CTA's shared memory
        // can go to another CTA
        for (int u = issued > kStages ? issued - kStages : 0; u < issued; ++u)
          mbar_wait_drain(&full[u % kStages], (u / kStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(kGemmBM, kGemmBN, 0, 1);
      // descriptor templates for stage 0 (start-address field = address >> 4)
      const uint64_t da = desc_sw128(smem_u32(smem), 16, 1024);
      const uint64_t db = desc_sw128(smem_u32(smem) + kABytes, kBBlockBytes, 1024);
      int stage = 0;
      uint32_t phase = 0;
      int acc_i = 0;
      for (int t = blockIdx.x; t < p.total_tiles && !*abort_flag; t += gridDim.x) {
        TileCoord tc;
        if (!decode_tile(p, t, tc)) continue;
        const GemmProblem& pr = p.prob[tc.prob];
        const int nk = (pr.K + kGemmBK - 1) / kGemmBK;
        const int buf = acc_i & 1;
        const uint32_t use = static_cast<uint32_t>(acc_i >> 1);
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * kAccStride;
        for (int kb = 0; kb < nk; kb += 2) {
          const bool two = kb + 1 < nk;
          // both stages' waits back to back, then their 8 MMAs in one burst
          if (!mbar_wait(&full[stage], phase, abort_flag)) break;
          const int stage2 = stage + 1 == kStages ? 0 : stage + 1;
          const uint32_t phase2 = stage + 1 == kStages ? phase ^ 1 : phase;
          if (two && !mbar_wait(&full[stage2], phase2, abort_flag)) break;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && !two) break;
            const int sth = h == 0 ? stage : stage2;
            const uint64_t ad = da + ((sth * kStageBytes) >> 4);
            const uint64_t bd = db + ((sth * kStageBytes) >> 4);
#pragma unroll
            for (int k = 0; k < kGemmBK / 16; ++k)
              mma_ss(d, ad + ((32 * k) >> 4), bd + ((2048 * k) >> 4), idesc,
                     (kb + h > 0 || k > 0) ? 1u : 0u);
            mma_commit(&empty[sth]);
          }
          const int adv = two ? 2 : 1;
          for (int a = 0; a < adv; ++a) {
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        mma_commit(&acc_full[buf]);
        ++acc_i;
      }
      if (*abort_flag) {
        // the MMAs this thread queued must finish before TMEM is freed
        mma_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
    __syncwarp();
  } else {
    const int q = warp & 3;   // TMEM lane quadrant this warp may access
    uint8_t* stg = staging + q * 2 * kChunkBytes;
    int acc_i = 0;
    int n_chunk = 0;          // chunks this warp has stored (staging slot = n_chunk & 1)
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      TileCoord tc;
      if (!decode_tile(p, t, tc)) continue;
      const GemmProblem& pr = p.prob[tc.prob];
      const int buf = acc_i & 1;
      const uint32_t use = static_cast<uint32_t>(acc_i >> 1);
      if (!mbar_wait(&acc_full[buf], use & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + buf * kAccStride + (static_cast<uint32_t>(32 * q) << 16);
      const int y = tc.m0 + 32 * q;
      const bool rows_in = y < pr.M;
#pragma unroll 1
      for (int c0 = 0; c0 < kGemmBN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(taddr + c0, r);
        tmem_wait_ld();
        if (c0 + 32 >= kGemmBN) {
          // the accumulator is free once its last columns are in registers
          tc_fence_before();
          mbar_arrive(&acc_empty[buf]);
        }
        const int x = tc.n0 + c0;
        if (!rows_in || x >= pr.N) continue;
        if (pr.softmax32) {
          // the chunk is one 32-column group (tiles start at multiples of 32):
          // p = 2^(v - max) / sum over the group, per row
          float m = __uint_as_float(r[0]);
#pragma unroll
          for (int j = 1; j < 32; ++j) m = fmaxf(m, __uint_as_float(r[j]));
          float sum = 0.f;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float e = exp2f(__uint_as_float(r[j]) - m);
            sum += e;
            r[j] = __float_as_uint(e);
          }
          const float inv = 1.0f / sum;
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * inv);
        }
        // the slot's previous store must have finished reading it
        if (lane == 0) bulk_wait_read<1>();
        __syncwarp();
        uint8_t* chunk = stg + (n_chunk & 1) * kChunkBytes;
        if (pr.out_f32) {
          // 128-byte rows, 16-byte unit j of row `lane` at j ^ (lane & 7)
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4*>(chunk + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
        } else {
          // 64-byte rows, 16-byte unit j of row `lane` at j ^ ((lane >> 1) & 3)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 v;
            v.x = pack_half2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
            v.y = pack_half2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
            v.z = pack_half2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
            v.w = pack_half2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
            *reinterpret_cast<uint4*>(chunk + lane * 64 + ((j ^ ((lane >> 1) & 3)) << 4)) = v;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&pr.c, chunk, x, y);
          bulk_commit_group();
        }
        ++n_chunk;
      }
      ++acc_i;
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && *abort_flag && p.status) atomicOr(p.status, DEV_TIMEOUT);
}

}  // namespace

int gemm_make_problem(GemmProblem* p, const void* a, int64_t lda, const void* b, int64_t ldb,
                      void* c, int64_t ldc, int M, int N, int K, const int32_t* pred,
                      bool out_f32) {
  if (M <= 0 || N <= 0 || K <= 0) return 1;
  if (N % 16 || K % 8 || lda % 8 || ldb % 8 || ldc % 8) return 1;   // 16-byte rows
  if (lda < K || ldb < N || ldc < N) return 1;
  if ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b) |
       reinterpret_cast<uintptr_t>(c)) & 15)
    return 1;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(lda) * 2};
    const uint32_t box[2] = {64, kGemmBM};
    if (encode_f16_tmap(&p->a, a, 2, dims, strides, box) != 0) return 2;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(K)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldb) * 2};
    const uint32_t box[2] = {64, 64};
    if (encode_f16_tmap(&p->b, b, 2, dims, strides, box) != 0) return 2;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
    const uint64_t strides[1] = {static_cast<uint64_t>(ldc) * (out_f32 ? 4 : 2)};
    const uint32_t box[2] = {32, 32};
    if (encode_tmap(&p->c, out_f32, c, 2, dims, strides, box, out_f32 ? 128 : 64) != 0) return 2;
  }
  p->out_f32 = out_f32 ? 1 : 0;
  p->softmax32 = 0;
  p->M = M;
  p->N = N;
  p->K = K;
  p->tiles_n = (N + kGemmBN - 1) / kGemmBN;
  p->pred = pred;
  return 0;
}

int gemm_set_softmax32(GemmProblem* p) {
  static_assert(kGemmBN % 32 == 0, "tiles start on 32-column groups");
  if (p->out_f32 || p->N % 32) return 1;
  p->softmax32 = 1;
  return 0;
}

int gemm_init() {
  // the shared-memory attribute is per device: set it once on each device used
  static std::mutex mu;
  static bool done[kMaxDevices] = {};
  const int dev = current_device();
  if (dev < 0) return 4;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(gemm_f16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess)
      return 4;
    done[dev] = true;
  }
  return 0;
}

int gemm_launch(GemmParams* params, cudaStream_t stream, int max_ctas) {
  if (gemm_init()) return 4;
  int total = 0;
  for (int i = 0; i < params->n_problems; ++i) {
    GemmProblem& pr = params->prob[i];
    const int tiles_m = (pr.M + kGemmBM - 1) / kGemmBM;
    pr.tile_begin = total;
    total += tiles_m * pr.tiles_n;
    pr.tile_end = total;
  }
  params->total_tiles = total;
  if (total == 0) return 0;
  int grid = total < max_ctas ? total : max_ctas;
  gemm_f16_kernel<<<grid, kThreads, kSmemBytes, stream>>>(*params);
  return cudaGetLastError() == cudaSuccess ? 0 : 4;
}

}  // namespace pl
