/*
 * pl.h — C ABI of the streaming pyramid denoising round (PersonaLive) on B200.
 *
 * One round, as the PersonaLive write-up (juhe.plus) describes it in
 * "流式金字塔去噪" (streaming pyramid denoising): a pile of 4 windows x 4
 * latent frames sits at DDIM timesteps {999, 666, 333, 0}; each round appends
 * a new noise window at t = 999, runs the 16 frames as one batch, moves every
 * window one DDIM step (step length 333) and pops the t = 0 window with its
 * predicted x0. Inside the batch every reference-attention layer attends over
 * the frame's own tokens concatenated with a reference KV bank of 1..4 entries
 * ("三条条件通路", three conditioning paths), next to a 32-token, 16-d motion
 * cross-attention. After the step the round's motion embeddings are checked
 * against a motion bank (minimum L2 distance > 17 appends an anchor, at most 3
 * times; "抗身份漂移的补丁", identity-drift guard).
 *
 * Conventions for every call:
 *  - Pointers named as device pointers must point to memory of the current
 *    CUDA device; the caller allocates and owns all of it (the library never
 *    allocates device memory). Host pointers are read before the call returns.
 *  - All fp16 matrices are row-major with the stated leading dimension in
 *    ELEMENTS; leading dimensions and frame strides must be multiples of 8
 *    (16 bytes) and device pointers 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream). Every call is
 *    asynchronous on it unless stated otherwise.
 *  - The return value reports host-side validation and launch errors only.
 *    Kernels that detect a problem on the device (a bounded wait that ran
 *    out, an argument outside the contract) set bits of a device status word
 *    instead of trapping. Calls on a context (pl_ctx, pl_sink, pl_lpm) use the
 *    context's word: pl_get_device_status() / the state getters read it.
 *    Calls without a context (pl_gemm_f16, pl_segment_attention,
 *    pl_pr_sink_attention, pl_ref_attention, pl_ref_attention_noalloc,
 *    pl_motion_xattn, pl_rope_attention) share one word per device:
 *    pl_get_call_status() reads and clears it. After such a report the output
 *    of the call that raised it is unspecified.
 *  - Nothing aborts, exits or traps. A context is not thread-safe.
 */
#ifndef PL_H_
#define PL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pl_status {
  PL_OK = 0,
  PL_EINVAL = 1,       /* an argument is outside its documented range */
  PL_ESTATE = 2,       /* call order violated (e.g. a round before pl_bank_init) */
  PL_ENOMEM = 3,       /* the caller's workspace is smaller than required */
  PL_ECUDA = 4,        /* a CUDA runtime/driver call failed */
  PL_ETIMEOUT = 5,     /* a device-side bounded wait gave up */
  PL_EDEVICE = 6,      /* a kernel flagged a contract violation on the device */
  PL_EUNSUPPORTED = 7  /* shape not supported by this build (e.g. head_dim) */
} pl_status;

/* Static description of a status code. Never NULL. */
const char* pl_status_string(int status);

/* ABI version of this header (incremented on any signature change). */
int pl_abi_version(void);

/* ------------------------------------------------------------------ *
 * Stateless primitives
 * ------------------------------------------------------------------ */

/* C[M,N] = A[M,K] * B[K,N] (fp16 in, fp32 accumulate, fp16 out) on tcgen05
 * tensor cores. a, b, c: device pointers; lda >= K, ldb >= N, ldc >= N.
 * Requires N % 16 == 0 and K % 8 == 0. Used for every projection of the
 * reference attention (Q/K/V/O) and of the motion cross-attention (Q/O). */
pl_status pl_gemm_f16(const void* a, int64_t lda, const void* b, int64_t ldb, void* c,
                      int64_t ldc, int M, int N, int K, void* stream);

/* One KV segment of an attention call. Row r of frame f of the segment's K
 * starts at element (f * frame_stride + r) * ld of `k` (same for `v`); head h
 * occupies columns [h * head_dim, (h + 1) * head_dim). frame_stride == 0
 * means the segment is shared by all frames (a reference bank entry). */
typedef struct pl_kv_segment {
  const void* k;          /* device, fp16 */
  const void* v;          /* device, fp16 */
  int64_t len;            /* rows (keys) in the segment, >= 1 */
  int64_t ld;             /* elements between rows, multiple of 8 */
  int64_t frame_stride;   /* elements between frames, multiple of 8, or 0 */
} pl_kv_segment;

/* Attention core over a list of KV segments, never materialising their
 * concatenation (PersonaLive write-up, "三条条件通路": own KV followed by the
 * reference bank; LiveAnimate page, PR-Sink: query block + sink + retrieved
 * block + rolling blocks):
 *   out[f, i, h] = softmax_j( q[f,i,h] . K_cat[f,j,h] / sqrt(head_dim) ) V_cat[f,j,h]
 * with K_cat/V_cat = segments in order. Full (non-causal) attention, fp32
 * softmax statistics, fp16 output.
 * q: device [frames][n_q][ldq] (frame stride q_frame_stride elements);
 * out: device, same addressing with ldo / out_frame_stride.
 * head_dim in {40, 64, 80, 128, 160}; 1 <= n_segs <= 8. */
pl_status pl_segment_attention(const void* q, int64_t ldq, int64_t q_frame_stride,
                               const pl_kv_segment* segs, int n_segs, int frames, int n_q,
                               int heads, int head_dim, void* out, int64_t ldo,
                               int64_t out_frame_stride, void* stream);

/* PR-Sink bounded attention of one block (LiveAnimate page, PR-Sink: a
 * bounded KV cache of a static sink block, one dynamic block retrieved by
 * pose and a rolling buffer of three slots; attention within the query block
 * is full, as in block-causal generation):
 *   j* = argmin_j ||pose_query - pose_store[j]||^2   (fp64, lowest j on ties)
 *   out = softmax(q K_cat^T / sqrt(head_dim)) V_cat,
 *   K_cat = [k_own ; k_sink ; k_pool[j*] ; k_roll[0..n_roll)] (V alike).
 * The retrieval runs on the device and feeds the attention directly (no host
 * round trip). q, every k / v, out: device fp16 [n][heads*head_dim];
 * k_pool / v_pool: device fp16 [n_pool][n][heads*head_dim]; pose_store:
 * device fp32 [n_pool][pose_dim]; pose_query: device fp32 [pose_dim];
 * k_roll / v_roll: host arrays of n_roll (0..5) device pointers; retrieved:
 * device int32 [1] (written: j*); retrieved_d2: device double [1] or NULL.
 * head_dim in {40, 64, 80, 128, 160}; 1 <= n_pool <= 65536. */
pl_status pl_pr_sink_attention(const void* q, const void* k_own, const void* v_own,
                               const void* k_sink, const void* v_sink, const void* k_pool,
                               const void* v_pool, int n_pool, const float* pose_store,
                               const float* pose_query, int pose_dim,
                               const void* const* k_roll, const void* const* v_roll,
                               int n_roll, int n, int heads, int head_dim, void* out,
                               int32_t* retrieved, double* retrieved_d2, void* stream);

/* Bytes of device workspace pl_ref_attention needs. */
pl_status pl_ref_attention_workspace_bytes(int frames, int n, int c, int n_bank,
                                           size_t* bytes);

/* One reference-attention layer (PersonaLive write-up, "三条条件通路"):
 *   Q = h Wq; K = [h ; bank_0 ; ...] Wk; V = [h ; bank_0 ; ...] Wv;
 *   out = attention(Q, K, V) Wo,  8-head split of C, scale 1/sqrt(C/heads).
 * hidden: device fp16 [frames][n][c]; w_qkv: device fp16 [c][3c] = [Wq|Wk|Wv];
 * w_o: device fp16 [c][c]; bank_feats: host array of n_bank device pointers,
 * each fp16 [n][c] (norm_hidden_states of the Reference UNet, shared by all
 * frames); out: device fp16 [frames][n][c]. 0 <= n_bank <= 4.
 * workspace: device, >= pl_ref_attention_workspace_bytes(). */
pl_status pl_ref_attention(const void* hidden, const void* w_qkv, const void* w_o,
                           const void* const* bank_feats, int n_bank, int frames, int n,
                           int c, int heads, void* out, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Scratch size behind pl_ref_attention_noalloc: 32 MiB per device. */
#define PL_NOALLOC_SCRATCH_BYTES (32u << 20)

/* pl_ref_attention without a workspace argument (no counterpart in the
 * pages: an interface convenience of this library).
 *
 * For callers that cannot allocate device memory: code embedded in a host
 * application that owns every device allocation, a real-time thread that must
 * not block in cudaMalloc/cudaFree (both may synchronise the device), or a
 * plugin with no allocator of its own. They still pass hidden, the weights,
 * the bank features and out, exactly as for pl_ref_attention; the
 * intermediate Q/K/V, bank K/V and pre-projection output go to a file-scope
 * device array of PL_NOALLOC_SCRATCH_BYTES instead of a caller workspace.
 *
 * - Problems whose pl_ref_attention_workspace_bytes exceeds
 *   PL_NOALLOC_SCRATCH_BYTES are rejected with PL_ENOMEM before any device
 *   work (e.g. the 16-frame 8x8/C1280 layer with one bank entry needs about
 *   11 MB and fits; a 64x64/C320 layer does not).
 * - The call allocates nothing. Its first call on a device looks up the
 *   array's device address (cudaGetSymbolAddress) and caches it, so make that
 *   first call outside any stream capture. Every device that has made a call
 *   keeps the array until the process exits. The cached address is not looked
 *   up again: no cudaDeviceReset may come between calls on a device.
 * - Device-side problems go to the context-free status word
 *   (pl_get_call_status), like those of pl_ref_attention.
 * - All calls share one array per device and it keeps the last call's
 *   contents; nothing in it has to start at zero. Calls whose execution can
 *   overlap on the GPU (other streams, other threads) race on the array:
 *   order them on one stream or synchronise between them. */
pl_status pl_ref_attention_noalloc(const void* hidden, const void* w_qkv, const void* w_o,
                                   const void* const* bank_feats, int n_bank, int frames,
                                   int n, int c, int heads, void* out, void* stream);

/* Bytes of device workspace pl_motion_xattn needs. */
pl_status pl_motion_xattn_workspace_bytes(int frames, int n, int c, size_t* bytes);

/* Motion cross-attention (PersonaLive write-up, "三条条件通路": the 512-d
 * expression embedding becomes 32 tokens x 16 channels plus a sinusoidal
 * position code; cross_attention_dim 16; 8 heads):
 *   tok[f] = reshape(motion[f], 32, 16) + PE  (PE[p,2i] = sin(p/10000^(2i/16)),
 *            PE[p,2i+1] = cos(same)), in fp32;
 *   out = softmax((x Mq)(tok Mk)^T / sqrt(c/heads)) (tok Mv) Mo,
 * with the tokens, tok Mk / tok Mv and x Mq kept in fp32 (the embedding's
 * magnitude grows along a stream, and fp16 there would be amplified by the
 * softmax); x and the attention output enter the projections as fp16.
 * x: device fp16 [frames][n][c]; motion: device fp32 [frames][512];
 * m_q, m_o: device fp16 [c][c]; m_kv: device fp16 [16][2c] = [Mk|Mv];
 * out: device fp16 [frames][n][c]. */
pl_status pl_motion_xattn(const void* x, const float* motion, const void* m_q,
                          const void* m_kv, const void* m_o, int frames, int n, int c,
                          int heads, void* out, void* workspace, size_t workspace_bytes,
                          void* stream);

/* Motion-bank check (PersonaLive write-up, "抗身份漂移的补丁"), in query
 * order: for query q, d2_j = ||q - bank_j||^2 (fp64) over the *count entries
 * present (including entries appended earlier in this call); argmin = lowest
 * index of the minimum; if d2_min > threshold^2 and *appends < cap and
 * *count < capacity, q is copied to bank[*count], ++*count, ++*appends.
 * bank: device fp32 [capacity][dim]; count, appends: device int32 (state,
 * read and updated on the device); queries: device fp32 [n_queries][dim];
 * argmin (int32), min_d2 (double), appended (uint8): device [n_queries],
 * each may be NULL. cap = 0 turns the call into a pure nearest-neighbour
 * retrieval (LiveAnimate page, PR-Sink's pose-retrieved dynamic sink).
 * 1 <= dim <= 4096, 1 <= capacity <= 2^24, 0 <= n_queries <= 64.
 * Banks of up to 32 entries checked with up to 32 queries run in one CTA
 * and need no workspace (workspace may be NULL). Larger ones read the bank
 * once for all queries across the GPU and keep per-CTA minima in a device
 * workspace of pl_motion_bank_check_workspace_bytes() (16-byte aligned;
 * PL_ENOMEM when smaller); they also need n_queries * dim <= 20480. */
pl_status pl_motion_bank_check_workspace_bytes(int capacity, int dim, int n_queries,
                                               size_t* bytes);
pl_status pl_motion_bank_check(float* bank, int32_t* count, int32_t* appends, int capacity,
                               int dim, const float* queries, int n_queries, float threshold,
                               int cap, int32_t* argmin, double* min_d2, uint8_t* appended,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of device workspace pl_nearest needs for a store of `count` entries. */
pl_status pl_nearest_workspace_bytes(int64_t count, size_t* bytes);

/* Nearest stored vector for large stores (LiveAnimate page, PR-Sink's pose
 * retrieval; the motion-bank distance of the PersonaLive write-up,
 * "抗身份漂移的补丁", without appends): argmin_j ||query - store_j||^2 with
 * fp64 distances, lowest j on equal distances, reading the store once over
 * the whole GPU. store: device fp32 [count][dim] (16-byte aligned rows when
 * dim % 4 == 0); query: device fp32 [dim]; argmin: device int64 [1];
 * min_d2: device double [1] or NULL; workspace: device, >=
 * pl_nearest_workspace_bytes(count). 1 <= count < 2^40, 1 <= dim <= 65536. */
pl_status pl_nearest(const float* store, int64_t count, int dim, const float* query,
                     int64_t* argmin, double* min_d2, void* workspace, size_t workspace_bytes,
                     void* stream);

/* ------------------------------------------------------------------ *
 * PR-Sink cache: the bounded KV cache of one block-streaming generator
 * ------------------------------------------------------------------ */

/* LiveAnimate page, PR-Sink: a bounded KV cache in three parts, the static
 * sink (the first generated block, kept for good), one dynamic block chosen
 * by pose from the history, and a rolling buffer of three slots; memory and
 * per-block cost stay constant however long the stream runs. Readings of
 * what the page leaves open: a block enters the rolling buffer after its own
 * step (the first block becomes the sink instead); the block a full rolling
 * buffer pushes out enters the pose pool with its pose descriptor; a full
 * pool replaces its oldest entry; the dynamic block is the pool entry
 * nearest to the current block's pose (squared L2 in fp64, lowest pool slot
 * on equal distances), attended only while the pool is not empty.
 *
 * One step: out = softmax(q K_cat^T / sqrt(head_dim)) V_cat over
 *   K_cat = [own ; sink ; rolling (oldest first) ; pool[j*]]   (V alike),
 * each part present once it exists; then the cache update above. Blocks
 * live in a device arena of pool_capacity + 5 blocks inside the caller's
 * workspace and never move: the sink, the rolling buffer and the pool are
 * index lists, so a step copies no K/V. The caller writes the current
 * block's K and V (fp16 [n][heads*head_dim]) at the pointers
 * pl_sink_block_kv returns, before pl_sink_step. */
typedef struct pl_sink pl_sink;

typedef struct pl_sink_state {
  int64_t blocks;         /* steps taken */
  int32_t has_sink;
  int32_t n_roll;         /* blocks in the rolling buffer (0..3) */
  int32_t pool_count;     /* entries in the pose pool */
  int32_t retrieved;      /* pool slot attended by the last step, -1 when none */
  double retrieved_d2;    /* its squared pose distance (0 when none) */
  uint32_t device_status;
} pl_sink_state;

pl_status pl_sink_workspace_bytes(int n, int heads, int head_dim, int pool_capacity,
                                  int pose_dim, size_t* bytes);
/* n tokens per block (>= 1), head_dim in {40, 64, 80, 128, 160},
 * 1 <= pool_capacity <= 4096, 1 <= pose_dim <= 4096; workspace: device,
 * 256-byte aligned, >= pl_sink_workspace_bytes. */
pl_status pl_sink_create(int n, int heads, int head_dim, int pool_capacity, int pose_dim,
                         void* workspace, size_t workspace_bytes, pl_sink** out);
pl_status pl_sink_destroy(pl_sink* sink);
/* Device pointers where the next block's K and V go (fp16 [n][heads*head_dim]). */
pl_status pl_sink_block_kv(pl_sink* sink, void** k, void** v);
/* One block: q, out device fp16 [n][heads*head_dim]; pose: device fp32
 * [pose_dim], the block's pose descriptor. */
pl_status pl_sink_step(pl_sink* sink, const void* q, const float* pose, void* out, void* stream);
/* Synchronise `stream` and report the cache state. */
pl_status pl_sink_get_state(pl_sink* sink, pl_sink_state* out, void* stream);

/* ------------------------------------------------------------------ *
 * Pre-rotary KV cache with a sliding window
 * ------------------------------------------------------------------ */

/* Rotary position table (the rotary code of the LPM 1.0 write-up, section
 * 7.4 "Pre-RoPE KV Cache"): tab[pos][i] = (cos, sin)(pos * base^(-2i / head_dim)),
 * i < head_dim / 2, fp32 pairs computed from fp64 angles. tab: device,
 * 8-byte aligned, positions * head_dim / 2 float pairs. */
pl_status pl_rope_table(float* tab, int positions, int head_dim, float base, void* stream);

/* Attention with the rotary code (LPM 1.0 write-up, section 7.4 "Pre-RoPE
 * KV Cache": K/V are kept before the rotary code, which is applied by each
 * token's position in the current window):
 *   out = softmax(R(q) R(K_cat)^T / sqrt(head_dim)) V_cat,
 * where R turns the pairs (2i, 2i+1) of each head by pos * theta_i; query
 * row g sits at q_pos0 + g, row j of segment s at seg_pos0[s] + j. Q and
 * every K are rotated once per key into the workspace (an HBM-bound pass),
 * then the segment attention runs on the rotated copies and the caller's V.
 * q, out: device fp16 [n_q][ld]; segments as pl_segment_attention with
 * frame_stride 0 and ld = heads * head_dim; tab: pl_rope_table covering every
 * position used; workspace: device, 16-byte aligned, >=
 * pl_rope_attention_workspace_bytes(n_q, total keys, heads, head_dim). */
pl_status pl_rope_attention_workspace_bytes(int n_q, int64_t total_keys, int heads, int head_dim,
                                            size_t* bytes);
pl_status pl_rope_attention(const void* q, int64_t ldq, int q_pos0, const pl_kv_segment* segs,
                            const int64_t* seg_pos0, int n_segs, int n_q, int heads, int head_dim,
                            const float* tab, int tab_positions, void* out, int64_t ldo,
                            void* workspace, size_t workspace_bytes, void* stream);

/* LPM window cache (LPM 1.0 write-up, section 7.3 "滑动窗口注意力"): a new
 * chunk attends the reference tokens (always kept), three fixed sink chunks and the two most
 * recent chunks, so the context stays bounded however long the session.
 * Readings of what the write-up leaves open: the first three chunks become
 * the sinks; later chunks slide (a full window drops its oldest); positions
 * are the order of [reference ; sinks ; sliding oldest first ; current] in
 * the window, so a sliding chunk's position changes as it ages and its
 * cached (un-rotated) K is rotated again at its new position; the reference
 * and the sinks never move and are rotated once. Chunks live in a device
 * arena of 6 chunk blocks and never
 * move; the caller writes each chunk's un-rotated K and V (fp16
 * [chunk_tokens][heads*head_dim]) at the pointers pl_lpm_chunk_kv returns,
 * and the reference tokens' once at pl_lpm_ref_kv's. */
typedef struct pl_lpm pl_lpm;

typedef struct pl_lpm_state {
  int64_t chunks;       /* steps taken */
  int32_t n_sink;       /* 0..3 */
  int32_t n_slide;      /* 0..2 */
  int32_t last_q_pos0;  /* window position of the last step's first query row, -1 before */
} pl_lpm_state;

pl_status pl_lpm_workspace_bytes(int ref_tokens, int chunk_tokens, int heads, int head_dim,
                                 size_t* bytes);
/* ref_tokens >= 0, chunk_tokens >= 1, head_dim in {40, 64, 80, 128, 160},
 * rope_base > 1;
 * workspace: device, 256-byte aligned. */
pl_status pl_lpm_create(int ref_tokens, int chunk_tokens, int heads, int head_dim,
                        float rope_base, void* workspace, size_t workspace_bytes, pl_lpm** out);
pl_status pl_lpm_destroy(pl_lpm* lpm);
pl_status pl_lpm_ref_kv(pl_lpm* lpm, void** k, void** v);
pl_status pl_lpm_chunk_kv(pl_lpm* lpm, void** k, void** v);
/* One chunk: q, out device fp16 [chunk_tokens][heads*head_dim] (un-rotated q). */
pl_status pl_lpm_step(pl_lpm* lpm, const void* q, void* out, void* stream);
pl_status pl_lpm_get_state(pl_lpm* lpm, pl_lpm_state* out);

/* ------------------------------------------------------------------ *
 * Pose path front
 * ------------------------------------------------------------------ */

/* PersonaLive write-up, "三条条件通路" (pose as a residual): 21 implicit 3D
 * keypoints with pitch / yaw / roll / translation / scale; retargeting keeps
 * the reference's canonical keypoints and scale and takes only the driving
 * frame's rotation and half its translation; 7 of the points are drawn as
 * coloured dots for the pose guider. Readings where the page is silent:
 * angles in degrees, R = Rz(roll) Ry(yaw) Rx(pitch) on column vectors,
 * keypoint = scale * R c + 0.5 t; the dot image is orthographic with x, y in
 * [-1, 1] mapped to [0, W] x [0, H]; a pixel (centre (x + 0.5, y + 0.5))
 * takes the colour of the last selected dot within `radius` pixels
 * (d^2 <= r^2 in fp64), black elsewhere; the 12 prefill frames' keypoints are
 * the 13-point ramp from the reference pose to the first driving pose, last
 * point dropped. Keypoints are fp64. */
#define PL_POSE_POINTS 21
#define PL_POSE_DOTS 7

/* kps[f][j] = scale * R(pose_f) canon[sel[j]] + 0.5 t_f. canon: device fp32
 * [21][3]; poses: device fp32 [frames][6] = (pitch, yaw, roll, tx, ty, tz);
 * sel: host int32 [7] (indices < 21); kps: device double [frames][7][3]. */
pl_status pl_pose_keypoints(const float* canon, float scale, const float* poses, int frames,
                            const int32_t* sel, double* kps, void* stream);
/* out[k] = from + (k / frames)(to - from), k < frames: the prefill ramp
 * (frames = 12). from, to: device double [7][3]; out: device [frames][7][3]. */
pl_status pl_pose_ramp(const double* kps_from, const double* kps_to, int frames, double* out,
                       void* stream);
/* Dot images: image device fp32 [frames][3][H][W] from kps [frames][7][3];
 * colours: host fp32 [7][3]. */
pl_status pl_pose_dots(const double* kps, int frames, const float* colours, float radius, int H,
                       int W, float* image, void* stream);

/* ------------------------------------------------------------------ *
 * Stream context: the device-resident pile and the reference bank
 * ------------------------------------------------------------------ */

typedef struct pl_ctx pl_ctx;

#define PL_MAX_LAYERS 16
#define PL_WINDOWS 4            /* temporal_adaptive_step */
#define PL_WINDOW_FRAMES 4      /* temporal_window_size */
#define PL_BATCH_FRAMES 16
#define PL_MOTION_DIM 512
#define PL_MAX_BANK 4           /* reference + up to 3 anchors */

typedef struct pl_config {
  int32_t latent_c;                      /* 4 */
  int32_t latent_h, latent_w;            /* 64 x 64 for 512 x 512 frames */
  int32_t n_layers;                      /* 0..16 reference-attention layers */
  int32_t layer_tokens[PL_MAX_LAYERS];   /* tokens per frame N_l */
  int32_t layer_channels[PL_MAX_LAYERS]; /* channels C_l (multiple of heads*8) */
  int32_t heads;                         /* 8 */
  float drift_threshold;                 /* 17 */
  int32_t append_cap;                    /* 3 (so the bank holds at most 4) */
  int32_t sessions;                      /* independent streams served together, 1..8
                                            (0 is read as 1); see below */
  int32_t motion_blocks;                 /* motion cross-attention blocks per layer:
                                            1 (0 is read as 1) or 2 (PersonaLive
                                            write-up, "三条条件通路": the motion
                                            module's attention blocks are
                                            [Spatial_Cross, Spatial_Cross]; block 2
                                            has its own weights, the same 32 tokens,
                                            and block 1's output as its queries) */
} pl_config;

/* Sessions. A context serves S = cfg.sessions independent streams (same
 * weights, separate piles, banks and states) in the same launches: one
 * round of every session is one pl_stream_round. Every per-stream buffer
 * argument of the calls below then carries a leading session dimension
 * [S] in front of the shape given (session s at offset s times the
 * per-session size); for S = 1 the shapes are exactly as written. */

/* Per-layer weights (device fp16, row-major [in][out]); kept by pointer, so
 * they must outlive the context. */
typedef struct pl_layer_weights {
  const void* w_qkv; /* [C][3C] = [Wq | Wk | Wv] */
  const void* w_o;   /* [C][C] */
  const void* m_q;   /* [C][C] motion query projection */
  const void* m_kv;  /* [16][2C] = [Mk | Mv] */
  const void* m_o;   /* [C][C] */
  const void* m2_q;  /* second motion block (motion_blocks == 2, else NULL): [C][C] */
  const void* m2_kv; /* [16][2C] */
  const void* m2_o;  /* [C][C] */
} pl_layer_weights;

/* Host-side snapshot of the context's state (pl_get_state). */
typedef struct pl_state {
  int32_t initialised;
  int32_t head;                 /* physical slot of the oldest window */
  int32_t slot_t[PL_WINDOWS];   /* timestep per physical slot, -1 = free */
  int64_t rounds;
  int64_t frames_in;
  int64_t frames_out;
  int32_t bank_count;           /* entries in the motion bank == KV bank entries */
  int32_t appends;              /* anchors appended so far (<= append_cap) */
  uint32_t device_status;       /* bits set by kernels (0 = clean) */
} pl_state;

/* Device workspace a context with this configuration needs. */
pl_status pl_workspace_bytes(const pl_config* cfg, size_t* bytes);

/* Create a context on the current device inside the caller's workspace
 * (device memory, >= pl_workspace_bytes, 256-byte aligned). The context
 * struct itself lives in host memory owned by the library. */
pl_status pl_ctx_create(const pl_config* cfg, void* workspace, size_t workspace_bytes,
                        pl_ctx** out);

/* Destroy (releases host memory and any captured CUDA graph). NULL is a no-op. */
pl_status pl_ctx_destroy(pl_ctx* ctx);

/* Reference fusion, also the control-plane reset (PersonaLive write-up,
 * "首帧怎么办" and the pause/reset remark of "在线链路"):
 *  - KV bank <- entry 0 = ref_feats[l] projected by each layer's Wk/Wv;
 *  - per layer, the products Wo Mq (and Mo Mq2 with two motion blocks),
 *    accumulated in fp32 and rounded once to fp16: no nonlinearity sits
 *    between the O projection and the next motion query projection, so the
 *    round applies them as one [C][C] projection;
 *  - motion bank <- [ref_motion], appends <- 0;
 *  - prefill: 3 windows at t = 0, 333, 666 (oldest first), window w frame j =
 *    sqrt(abar_t) ref_latent + sqrt(1 - abar_t) prefill_eps[4w + j], with the
 *    12 frames' motion = ref + (k/12)(drive0 - ref), k = 0..11.
 * weights: host array [n_layers]; ref_feats: host array of n_layers device
 * fp16 [N_l][C_l]; anchor_feats: host array of 3*n_layers device pointers
 * (anchor a = 1..3, layer l at index (a-1)*n_layers + l) standing in for the
 * Reference UNet re-run of an anchor frame, or NULL (then appends extend only
 * the motion bank and the KV bank keeps entry 0). ref_motion, drive0_motion:
 * device fp32 [512]; ref_latent: device fp32 [4][H][W]; prefill_eps: device
 * fp32 [12][4][H][W]. All pointers must stay valid for the context's life. */
pl_status pl_bank_init(pl_ctx* ctx, const pl_layer_weights* weights,
                       const void* const* ref_feats, const void* const* anchor_feats,
                       const float* ref_motion, const float* drive0_motion,
                       const float* ref_latent, const float* prefill_eps, void* stream);

/* Append the new window (pure noise at t = 999) into the free slot.
 * new_noise: device fp32 [4][4][H][W]; new_motion: device fp32 [4][512]. */
pl_status pl_ring_push(pl_ctx* ctx, const float* new_noise, const float* new_motion,
                       void* stream);

/* One DDIM step (eta = 0, epsilon prediction, SD scaled-linear betas
 * 0.00085..0.012 over 1000 steps, step length 333) of every window of the
 * full pile, then the pop: out_x0 <- x0 of the t = 0 window, its slot freed.
 * eps: device fp32 [16][4][H][W] in batch order (oldest window first);
 * out_x0: device fp32 [4][4][H][W]. Requires a full pile (after pl_ring_push). */
pl_status pl_pyramid_ddim_step(pl_ctx* ctx, const float* eps, float* out_x0, void* stream);

/* pl_motion_bank_check on the context's motion bank with its threshold and
 * cap. When an append happens and anchor features were given, the anchor's
 * K/V are projected for every layer into the next KV-bank entry. */
pl_status pl_ctx_bank_check(pl_ctx* ctx, const float* queries, int n_queries,
                            int32_t* argmin, double* min_d2, uint8_t* appended,
                            void* stream);

/* One whole round: ring push, the n_layers reference-attention + motion
 * cross-attention layers on the 16-frame batch, the pyramid DDIM step with
 * pop, and the bank check of the 4 new motion embeddings.
 * hidden: host array [n_layers] of device fp16 [16][N_l][C_l] (batch order);
 * eps: device fp32 [16][4][H][W]; out_frames: device fp32 [4][4][H][W];
 * appended: device uint8 [4] or NULL; layer_out: host array [n_layers] of
 * device fp16 [16][N_l][C_l] or NULL (outputs then go to workspace);
 * attn_out: host array [n_layers] of device fp16 [16][N_l][C_l] or NULL:
 * when given, each layer's reference-attention sub-layer output (before the
 * motion cross-attention) is written there, and the round then applies Wo
 * and Mq (and Mo, Mq2) as separate projections instead of their products.
 * Layers of 1024 tokens per frame and more evaluate the motion
 * cross-attention per head as scores x (Mq K^T / sqrt(hd)) and output
 * P (V Mo) (the same function; fp16 roundings of those products).
 * The round is recorded as a CUDA graph on the first call and replayed while
 * the pointer arguments stay the same; inside the graph the layers run on
 * two streams the context owns, forked from and joined back into `stream`,
 * so the whole round is ordered on `stream` like any other call. */
pl_status pl_stream_round(pl_ctx* ctx, const float* new_noise, const float* new_motion,
                          const void* const* hidden, const float* eps, float* out_frames,
                          uint8_t* appended, void* const* layer_out,
                          void* const* attn_out, void* stream);

/* Host-buffer round: the serving boundary of the PersonaLive write-up,
 * "在线链路" (frames arrive from the host, four at a time, one forward per
 * four, decoded frames go back to the host), overlapped in the manner of the
 * LPM 1.0 page, section 7.5 (the steady rate is that of the slowest stage, so
 * the transfer of round k + 1 runs under the compute of round k).
 *
 * pl_host_staging_bytes: device staging the host path needs: two sets, each
 * holding one round's inputs and its x0 frames (about 2 x 0.4 GB per session
 * at the 512 x 512 geometry).
 *
 * pl_stream_round_host: the same round as pl_stream_round with
 * h_noise [S][4][4][H][W] fp32, h_motion [S][4][512] fp32, h_hidden (host
 * array [n_layers] of host fp16 [S][16][N_l][C_l]) and h_eps
 * [S][16][4][H][W] fp32 in host memory, and the x0 frames returned to
 * h_out_frames [S][4][4][H][W] fp32 in host memory. The inputs are copied on
 * a copy stream the context owns into staging set (call count mod 2) of
 * `staging` (device, 256-byte aligned, >= pl_host_staging_bytes, owned by the
 * caller and used by nothing else while the context lives), the round then
 * runs on `stream` and the frames are copied back on `stream`. Asynchronous
 * like cudaMemcpyAsync: the host buffers must be pinned for the copies to
 * overlap (pageable memory works but serialises), must stay unchanged until
 * the call's work is done, and h_out_frames is valid once `stream` has been
 * synchronised. Returns PL_EINVAL for a NULL or misaligned argument,
 * PL_ENOMEM for too small a staging buffer, PL_ESTATE before pl_bank_init,
 * PL_ECUDA when a copy or launch fails to enqueue. */
pl_status pl_host_staging_bytes(const pl_config* cfg, size_t* bytes);
pl_status pl_stream_round_host(pl_ctx* ctx, void* staging, size_t staging_bytes,
                               const float* h_noise, const float* h_motion,
                               const void* const* h_hidden, const float* h_eps,
                               float* h_out_frames, void* stream);

/* Synchronise `stream` and copy the state of session 0 to *out. */
pl_status pl_get_state(pl_ctx* ctx, pl_state* out, void* stream);

/* The same for session `session` (0 <= session < S). */
pl_status pl_get_session_state(pl_ctx* ctx, int session, pl_state* out, void* stream);

/* Synchronise `stream`, copy the motion bank (fp32 [count][512]) of session
 * 0 to host. */
pl_status pl_get_motion_bank(pl_ctx* ctx, float* host_out, int32_t* count, void* stream);

/* The same for session `session`. */
pl_status pl_get_session_motion_bank(pl_ctx* ctx, int session, float* host_out, int32_t* count,
                                     void* stream);

/* Synchronise `stream` and map the device status words of all sessions to a
 * status: PL_OK, PL_ETIMEOUT or PL_EDEVICE. Clears the words. */
pl_status pl_get_device_status(pl_ctx* ctx, void* stream);

/* Per-layer timing (no counterpart in the pages). With profiling on (this
 * call, or PL_PROFILE=1 in the environment when the context is created),
 * pl_stream_round runs the round outside its captured graph with a CUDA
 * event before each layer and after the last; pl_get_layer_ms synchronises
 * on the last event and writes the n_layers layer times (reference attention
 * plus motion cross-attention, ms) of the latest profiled round to ms_out
 * (host, n >= n_layers), or returns PL_ESTATE when there is none. The
 * events cost a few microseconds per layer; the graph path is unaffected
 * when profiling is off. */
pl_status pl_set_profiling(pl_ctx* ctx, int on);
pl_status pl_get_layer_ms(pl_ctx* ctx, float* ms_out, int n);

/* Kernels in the captured graph of the latest round that ran from a capture
 * (pl_stream_round with profiling off, or pl_stream_round_host): every
 * kernel of this library that one round launches, counted from the graph's
 * nodes when it was captured. *count (host); PL_ESTATE when no round has run
 * from a capture yet. */
pl_status pl_round_kernel_count(const pl_ctx* ctx, int* count);

/* Checkpoint and resume of the streams' state (no counterpart in the pages,
 * which pause and reset a stream but do not resume one; the state is small
 * and device-resident, so it is the natural unit to save).
 * pl_state_bytes: host bytes of a snapshot: a header, then per session the
 * device state (pile head, slot timesteps, bank count, appends, counters),
 * the pile's latents [16][latent_c][H][W] fp32, the slots' motion
 * embeddings [16][512] and the motion bank [capacity][512].
 * pl_state_export: synchronise `stream` and copy the snapshot to host_out
 * (host memory of >= pl_state_bytes; PL_ESTATE before pl_bank_init).
 * pl_state_import: restore a snapshot into a context of the same
 * configuration after its pl_bank_init (weights, reference and anchor
 * features given again): the header and every state are checked on the host
 * (PL_EINVAL on any mismatch, nothing written then); the KV-bank rows of the
 * appended anchors are projected again from the anchor features instead of
 * being stored. Rounds after an import continue the exported stream: same
 * inputs give the same outputs, bit for bit. Both calls block. */
pl_status pl_state_bytes(const pl_ctx* ctx, size_t* bytes);
pl_status pl_state_export(pl_ctx* ctx, void* host_out, size_t bytes, void* stream);
pl_status pl_state_import(pl_ctx* ctx, const void* host_in, size_t bytes, void* stream);

/* Synchronise `stream`, then read and clear the current device's status word
 * of context-free calls (see the conventions above): PL_OK, PL_ETIMEOUT (a
 * bounded wait gave up) or PL_EDEVICE (a kernel refused its arguments). The
 * word is shared by every context-free call on the device, from any stream
 * or thread, so a report covers all of them since the last read. The first
 * context-free call on a device (or pl_ctx_create) looks the word's address
 * up; make it outside stream capture. */
pl_status pl_get_call_status(void* stream);

/* ------------------------------------------------------------------ *
 * Test hooks (no counterpart in the pages): planted device-side failures
 * that exercise the error paths without faulting or hanging the GPU.
 * ------------------------------------------------------------------ */

#define PL_TEST_NO_KV 1    /* the producer loads Q but no K/V tile */
#define PL_TEST_BAD_BOX 2  /* the kernel is told a K/V box that is not its tile */

/* pl_segment_attention with a planted failure. PL_TEST_NO_KV: no K/V copy is
 * started, so the MMA issuers' bounded waits run out after wait_us
 * microseconds (1..2000000); the kernel raises its abort flag, every role
 * leaves its loop, TMEM is freed and the call status becomes PL_ETIMEOUT.
 * PL_TEST_BAD_BOX: the box count the kernel checks is off by 16 rows (the
 * tensor maps themselves are right), so every CTA returns before any copy
 * and the call status becomes PL_EDEVICE. `out` is not written in either
 * mode. Arguments as for pl_segment_attention. */
pl_status pl_test_segment_attention_fault(const void* q, int64_t ldq, int64_t q_frame_stride,
                                         const pl_kv_segment* segs, int n_segs, int frames,
                                         int n_q, int heads, int head_dim, void* out,
                                         int64_t ldo, int64_t out_frame_stride, int mode,
                                         uint32_t wait_us, void* stream);

/* Device pointer of the piles' latents, fp32 [S][4 slots][4][4][H][W]
 * (read-only view for tests; slot s holds the window at timestep slot_t[s]). */
const float* pl_ctx_ring_latents(const pl_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* PL_H_ */
