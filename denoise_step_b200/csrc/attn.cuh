// Flash-style attention over a list of KV segments on tcgen05 tensor cores.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace pl {

constexpr int kAttnMaxSegs = 8;

struct AttnSeg {
  CUtensorMap k;   // 4D {head_dim, heads, len, frames|1}, box {64, 1, BN, 1}
  CUtensorMap v;
  int len;
  int per_frame;   // 1: frame f reads its own rows, 0: shared by all frames
  const int32_t* block_sel;  // when non-null: every frame reads block *block_sel
                             // of a stacked segment (a retrieved cache block)
  int n_blocks;              // blocks in a stacked segment
  int frame_div;             // when > 0: frame f reads block f / frame_div of a stacked
                             // segment (one block per session of frame_div frames)
};

struct AttnParams {
  CUtensorMap q;               // 4D {head_dim, heads, n_q, frames}, box {64, 1, 128, 1}
  AttnSeg seg[kAttnMaxSegs];
  int n_fixed;                 // segments always attended
  int n_total;                 // segments available
  const int32_t* n_extra;      // when non-null: attend n_fixed + min(e, n_total - n_fixed) with
                               // e = n_extra[(frame / extra_div) * extra_stride]
  int extra_div, extra_stride; // frames per session and int32 stride between sessions' counts
  __half* out;
  int64_t ldo, out_fstride;
  int n_q, heads, frames;
  float scale_log2;            // log2(e) / sqrt(head_dim)
  int box_rows;                // K/V tensor-map box rows; must equal the kernel's key tile
  uint32_t* status;
  uint64_t wait_ns;            // limit of each bounded mbarrier wait (ns)
  int test_mode;               // 0, or kTestNoKV (a planted failure for tests)
};

// Test hook: the producer loads Q but no K/V tile, so the MMA issuers'
// bounded waits run out (nothing is in flight when they do).
constexpr int kTestNoKV = 1;

struct AttnSegHost {
  const void* k;
  const void* v;
  int64_t len, ld, frame_stride;
  // optional: `n_blocks` blocks stacked at `frame_stride`, the one attended
  // chosen on the device by *block_sel (0 <= *block_sel < n_blocks)
  int64_t n_blocks = 0;
  const int32_t* block_sel = nullptr;
  // optional: `n_blocks` blocks stacked at `frame_stride`, frame f reading
  // block f / frame_div (frame_div > 0; excludes block_sel)
  int frame_div = 0;
};

// Build params (tensor maps) on the host. Returns 0 on success.
int attn_make_params(AttnParams* p, const void* q, int64_t ldq, int64_t q_fstride,
                     const AttnSegHost* segs, int n_segs, int frames, int n_q, int heads,
                     int head_dim, void* out, int64_t ldo, int64_t out_fstride);
// Set kernel attributes once (call outside stream capture). 0 on success.
int attn_init();
int attn_launch(const AttnParams& p, int head_dim, cudaStream_t stream);

}  // namespace pl
