// PR-Sink cache (LiveAnimate page, PR-Sink): a bounded KV cache made of the
// static sink (first block), a rolling buffer of three blocks and a pose pool
// from which one block is retrieved per step by its pose descriptor.
//
// Blocks live in a fixed device arena and never move; the sink, the rolling
// buffer and the pool are index lists kept on the host (their evolution does
// not depend on data, only on the step count), so a step copies no K/V. The
// one data-dependent choice, the retrieved pool entry, is made on the device
// (nearest-descriptor search) and reaches the attention through a device
// block index, with no host round trip.
#include <cuda_runtime.h>

#include <cstring>
#include <new>
#include <vector>

#include "../../include/pl.h"
#include "attn.cuh"
#include "misc.cuh"
#include "ptx.cuh"

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
constexpr int kRoll = 3;     // rolling-buffer slots
constexpr int kMaxPool = 4096;

bool head_dim_ok(int hd) { return hd == 40 || hd == 64 || hd == 80 || hd == 128 || hd == 160; }

// physical arena block of the retrieved pool slot
__global__ void sink_select_kernel(const int32_t* __restrict__ pool_blk,
                                   const int32_t* __restrict__ argmin, int pool_count,
                                   int32_t* sel, uint32_t* status) {
  int a = *argmin;
  if (a < 0 || a >= pool_count) {
    atomicOr(status, pl::DEV_BADARG);
    a = 0;
  }
  *sel = pool_blk[a];
}

// desc_blk[block] <- pose; when a rolling block leaves for the pool:
// pool_desc[slot] <- desc_blk[evicted], pool_blk[slot] <- evicted
__global__ void sink_commit_kernel(float* desc_blk, const float* __restrict__ pose, int dim,
                                   int block, float* pool_desc, int32_t* pool_blk, int evicted,
                                   int slot) {
  for (int i = threadIdx.x; i < dim; i += blockDim.x)
    desc_blk[static_cast<int64_t>(block) * dim + i] = pose[i];
  if (evicted >= 0) {
    for (int i = threadIdx.x; i < dim; i += blockDim.x)
      pool_desc[static_cast<int64_t>(slot) * dim + i] =
          desc_blk[static_cast<int64_t>(evicted) * dim + i];
    if (threadIdx.x == 0) pool_blk[slot] = evicted;
  }
}

struct Layout {
  size_t k, v, desc, pool_desc, pool_blk, scratch, total;
};

Layout layout(int n, int heads, int hd, int pool, int dim) {
  const int64_t blocks = pool + kRoll + 2;
  const size_t be = static_cast<size_t>(n) * heads * hd;
  Layout l;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
  l.k = take(2 * blocks * be);
  l.v = take(2 * blocks * be);
  l.desc = take(4 * static_cast<size_t>(blocks) * dim);
  l.pool_desc = take(4 * static_cast<size_t>(pool) * dim);
  l.pool_blk = take(4 * static_cast<size_t>(pool));
  l.scratch = take(64);
  l.total = off;
  return l;
}

pl_status validate(int n, int heads, int hd, int pool, int dim) {
  if (n < 1 || heads < 1 || heads > 65535 || pool < 1 || pool > kMaxPool || dim < 1 || dim > 4096)
    return PL_EINVAL;
  if (!head_dim_ok(hd)) return PL_EUNSUPPORTED;
  if (static_cast<int64_t>(n) * heads * hd > (1ll << 40)) return PL_EINVAL;
  return PL_OK;
}

}  // namespace

struct pl_sink {
  int n, heads, hd, pool, dim, blocks;
  int64_t block_elems;
  __half* k_arena;
  __half* v_arena;
  float* desc_blk;
  float* pool_desc;
  int32_t* pool_blk;
  int32_t* argmin;
  double* d2;
  int32_t* sel;
  uint32_t* status;
  // index lists (host)
  int64_t steps;
  int sink_blk;
  int roll[kRoll];
  int n_roll;
  std::vector<int> pool_of_slot;
  int pool_count, pool_head;
  std::vector<int> free_blocks;
  int reserved;
  bool last_retrieved;
};

extern "C" {

pl_status pl_sink_workspace_bytes(int n, int heads, int head_dim, int pool_capacity,
                                  int pose_dim, size_t* bytes) {
  if (!bytes) return PL_EINVAL;
  const pl_status v = validate(n, heads, head_dim, pool_capacity, pose_dim);
  if (v) return v;
  *bytes = layout(n, heads, head_dim, pool_capacity, pose_dim).total;
  return PL_OK;
}

pl_status pl_sink_create(int n, int heads, int head_dim, int pool_capacity, int pose_dim,
                         void* workspace, size_t workspace_bytes, pl_sink** out) {
  if (!out || !workspace) return PL_EINVAL;
  *out = nullptr;
  const pl_status v = validate(n, heads, head_dim, pool_capacity, pose_dim);
  if (v) return v;
  if (reinterpret_cast<uintptr_t>(workspace) % kAlign) return PL_EINVAL;
  const Layout l = layout(n, heads, head_dim, pool_capacity, pose_dim);
  if (workspace_bytes < l.total) return PL_ENOMEM;
  pl_sink* s = new (std::nothrow) pl_sink;
  if (!s) return PL_ENOMEM;
  uint8_t* w = static_cast<uint8_t*>(workspace);
  s->n = n;
  s->heads = heads;
  s->hd = head_dim;
  s->pool = pool_capacity;
  s->dim = pose_dim;
  s->blocks = pool_capacity + kRoll + 2;
  s->block_elems = static_cast<int64_t>(n) * heads * head_dim;
  s->k_arena = reinterpret_cast<__half*>(w + l.k);
  s->v_arena = reinterpret_cast<__half*>(w + l.v);
  s->desc_blk = reinterpret_cast<float*>(w + l.desc);
  s->pool_desc = reinterpret_cast<float*>(w + l.pool_desc);
  s->pool_blk = reinterpret_cast<int32_t*>(w + l.pool_blk);
  uint8_t* sc = w + l.scratch;
  s->d2 = reinterpret_cast<double*>(sc);
  s->argmin = reinterpret_cast<int32_t*>(sc + 8);
  s->sel = reinterpret_cast<int32_t*>(sc + 12);
  s->status = reinterpret_cast<uint32_t*>(sc + 16);
  s->steps = 0;
  s->sink_blk = -1;
  s->n_roll = 0;
  s->pool_of_slot.assign(pool_capacity, -1);
  s->pool_count = 0;
  s->pool_head = 0;
  s->free_blocks.clear();
  for (int b = s->blocks - 1; b >= 0; --b) s->free_blocks.push_back(b);   // block 0 first
  s->reserved = -1;
  s->last_retrieved = false;
  if (cudaMemset(sc, 0, 64) != cudaSuccess || pl::attn_init() != 0) {
    delete s;
    return PL_ECUDA;
  }
  *out = s;
  return PL_OK;
}

pl_status pl_sink_destroy(pl_sink* sink) {
  delete sink;
  return PL_OK;
}

pl_status pl_sink_block_kv(pl_sink* s, void** k, void** v) {
  if (!s || !k || !v) return PL_EINVAL;
  if (s->reserved < 0) {
    if (s->free_blocks.empty()) return PL_ESTATE;   // cannot happen: blocks = pool + 5
    s->reserved = s->free_blocks.back();
    s->free_blocks.pop_back();
  }
  *k = s->k_arena + s->reserved * s->block_elems;
  *v = s->v_arena + s->reserved * s->block_elems;
  return PL_OK;
}

pl_status pl_sink_step(pl_sink* s, const void* q, const float* pose, void* out, void* stream) {
  if (!s || !q || !pose || !out) return PL_EINVAL;
  if (s->reserved < 0) return PL_ESTATE;   // the block's K/V were never placed
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(out)) & 15) return PL_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int64_t ld = static_cast<int64_t>(s->heads) * s->hd;
  auto seg_of = [&](int b) {
    return pl::AttnSegHost{s->k_arena + b * s->block_elems, s->v_arena + b * s->block_elems, s->n,
                           ld, 0};
  };
  pl::AttnSegHost segs[pl::kAttnMaxSegs];
  int ns = 0;
  segs[ns++] = seg_of(s->reserved);
  if (s->sink_blk >= 0) segs[ns++] = seg_of(s->sink_blk);
  for (int r = 0; r < s->n_roll; ++r) segs[ns++] = seg_of(s->roll[r]);
  const bool retrieve = s->pool_count > 0;
  if (retrieve) {
    pl::AttnSegHost pool{s->k_arena, s->v_arena, s->n, ld, s->block_elems};
    pool.n_blocks = s->blocks;
    pool.block_sel = s->sel;
    segs[ns++] = pool;
  }
  pl::AttnParams p;
  const int mr = pl::attn_make_params(&p, q, ld, s->block_elems, segs, ns, 1, s->n, s->heads, s->hd,
                                      out, ld, s->block_elems);
  if (mr) return mr == 1 ? PL_EINVAL : PL_ECUDA;
  p.status = s->status;
  if (retrieve) {
    if (pl::launch_nearest(s->pool_desc, s->pool_count, s->dim, pose, s->argmin, s->d2, st) !=
        cudaSuccess)
      return PL_ECUDA;
    sink_select_kernel<<<1, 1, 0, st>>>(s->pool_blk, s->argmin, s->pool_count, s->sel, s->status);
    if (cudaGetLastError() != cudaSuccess) return PL_ECUDA;
  }
  const int lr = pl::attn_launch(p, s->hd, st);
  if (lr) return lr == 7 ? PL_EUNSUPPORTED : PL_ECUDA;
  // cache update: the block becomes the sink, or enters the rolling buffer
  // (a full buffer hands its oldest block to the pool; a full pool drops
  // its oldest entry, whose arena block is free again)
  int evicted = -1, slot = -1;
  if (s->sink_blk < 0) {
    s->sink_blk = s->reserved;
  } else {
    if (s->n_roll == kRoll) {
      evicted = s->roll[0];
      for (int r = 1; r < kRoll; ++r) s->roll[r - 1] = s->roll[r];
      s->n_roll = kRoll - 1;
      if (s->pool_count < s->pool) {
        slot = s->pool_count++;
      } else {
        slot = s->pool_head;
        s->free_blocks.push_back(s->pool_of_slot[slot]);
        s->pool_head = (s->pool_head + 1) % s->pool;
      }
      s->pool_of_slot[slot] = evicted;
    }
    s->roll[s->n_roll++] = s->reserved;
  }
  sink_commit_kernel<<<1, 256, 0, st>>>(s->desc_blk, pose, s->dim, s->reserved, s->pool_desc,
                                        s->pool_blk, evicted, slot);
  if (cudaGetLastError() != cudaSuccess) return PL_ECUDA;
  s->reserved = -1;
  s->last_retrieved = retrieve;
  ++s->steps;
  return PL_OK;
}

pl_status pl_sink_get_state(pl_sink* s, pl_sink_state* out, void* stream) {
  if (!s || !out) return PL_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PL_ECUDA;
  std::memset(out, 0, sizeof(*out));
  out->blocks = s->steps;
  out->has_sink = s->sink_blk >= 0 ? 1 : 0;
  out->n_roll = s->n_roll;
  out->pool_count = s->pool_count;
  out->retrieved = -1;
  if (s->last_retrieved) {
    int32_t a = -1;
    double d = 0.0;
    if (cudaMemcpy(&a, s->argmin, sizeof(a), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemcpy(&d, s->d2, sizeof(d), cudaMemcpyDeviceToHost) != cudaSuccess)
      return PL_ECUDA;
    out->retrieved = a;
    out->retrieved_d2 = d;
  }
  uint32_t w = 0;
  if (cudaMemcpy(&w, s->status, sizeof(w), cudaMemcpyDeviceToHost) != cudaSuccess)
    return PL_ECUDA;
  out->device_status = w;
  return PL_OK;
}

}  // extern "C"
