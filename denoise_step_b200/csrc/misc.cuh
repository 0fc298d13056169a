// Streaming kernels of the round: pile (ring) maintenance, the pyramid DDIM
// step, the motion-bank check and the motion cross-attention pieces.
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace pl {

// Device-resident state of one stream (lives in the context's workspace).
struct DevState {
  int32_t head;            // physical slot of the oldest window
  int32_t slot_t[4];       // timestep per slot, -1 = free
  int32_t bank_count;      // motion-bank entries
  int32_t appends;         // anchors appended so far
  int32_t kv_extra;        // KV-bank entries beyond the reference (anchors projected)
  int32_t anchor_fire[4];  // [a] = 1 when anchor a was appended by the latest bank check
  int32_t initialised;
  int32_t pad_;
  int64_t rounds, frames_in, frames_out;
  uint32_t status;
  uint32_t pad2_[3];
};
// States of several sessions sit in an array; kernels step through it by
// whole int32 words (the attention reads appends at a fixed word stride).
static_assert(sizeof(DevState) % sizeof(int32_t) == 0 && sizeof(DevState) % 8 == 0,
              "DevState array stride");

// Per-timestep DDIM coefficients for the 4 timesteps of the table, in table
// order t = 999, 666, 333, 0: c = {1/sqrt(abar_t), sqrt(1-abar_t),
// sqrt(abar_prev), sqrt(1-abar_prev)} with abar_prev = 1 below t = 0, and
// fwd = {sqrt(abar_t), sqrt(1-abar_t)} for forward noising (the prefill).
struct DdimCoef {
  double c[4][4];
  double fwd[4][2];
};

// Host: fill the coefficients from the SD scaled-linear schedule.
void ddim_coefficients(DdimCoef* out);

// Host launchers. frame_elems = latent_c * H * W (multiple of 4). With
// `sessions` > 1 every buffer (and the DevState array) carries a leading
// session dimension: ring [S][16][fe], slot/batch motion [S][16][512], bank
// [S][capacity][512], per-call inputs [S][...]; one grid slice per session.
cudaError_t launch_prefill(DevState* st, float* ring, float* slot_motion, float* bank,
                           const float* ref_latent, const float* prefill_eps,
                           const float* ref_motion, const float* drive0, int64_t frame_elems,
                           int capacity, int sessions, cudaStream_t s);
cudaError_t launch_ring_push(DevState* st, float* ring, float* slot_motion, float* batch_motion,
                             const float* new_noise, const float* new_motion,
                             int64_t frame_elems, int sessions, cudaStream_t s);
cudaError_t launch_ddim(DevState* st, float* ring, const float* eps, float* out_x0,
                        int64_t frame_elems, const DdimCoef& coef, int sessions, cudaStream_t s);
cudaError_t launch_ring_commit(DevState* st, int sessions, cudaStream_t s);
// In-order motion-bank check. With st != null the counts live in st[session]
// and `count`/`appends` are ignored (capacity and queries <= 32: the one-CTA
// path); without it (a standalone bank) sessions must be 1, and banks past 32
// entries or 32 queries take the multi-CTA path, which needs a device
// workspace of bank_workspace_bytes() (0 for the one-CTA path). nq <= 64.
size_t bank_workspace_bytes(int64_t capacity, int nq);
cudaError_t launch_bank_check(float* bank, int32_t* count, int32_t* appends, int capacity,
                              int dim, const float* queries, int nq, double thr2, int cap,
                              int32_t* argmin, double* min_d2, uint8_t* appended,
                              DevState* st, int sessions, void* workspace, cudaStream_t s);
// argmin_j ||query - store_j||^2 over `count` stored vectors (fp64, lowest index on ties).
cudaError_t launch_nearest(const float* store, int count, int dim, const float* query,
                           int32_t* argmin, double* min_d2, cudaStream_t s);
// Nearest stored vector over a large store in one read: per-CTA partial
// minima (parts of them, in caller memory), then a one-CTA reduction.
int nearest_parts(int64_t count);
cudaError_t launch_nearest_large(const float* store, int64_t count, int dim, const float* query,
                                 double* part_d2, int64_t* part_idx, int parts, int64_t* argmin,
                                 double* min_d2, cudaStream_t s);
// Motion K/V (fp32 [F][32][2C]) of every frame from tokens = motion + PE (fp32).
cudaError_t launch_motion_kv(const float* motion, const __half* m_kv, int F, int C, float* kv,
                             cudaStream_t s);
// out[f*N + n][h*hd + d] = softmax_j(q . k_j / sqrt(hd)) v_j, 32 keys per frame;
// q fp32 (the Mq projection's fp32 accumulators), K/V fp32, out fp16.
cudaError_t launch_motion_attn(const float* q, int64_t ldq, const float* kv, int F, int N,
                               int C, int heads, __half* out, int64_t ldo, cudaStream_t s);
// Folded motion cross-attention weights of every frame and head (see
// motion_fold_kernel): W_qk fp16 [F][C][32 heads] (scores in base 2) and VM
// fp16 [F][32 heads][C], from K/V (fp32 [F][32][2C]), Wq and Mo (fp16 [C][C]).
cudaError_t launch_motion_fold(const float* kv, const __half* wq, const __half* mo, int F, int C,
                               int heads, __half* wqk, __half* vm, cudaStream_t s);

}  // namespace pl
