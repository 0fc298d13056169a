// Grouped fp16 GEMM on tcgen05 tensor cores: C[M,N] = A[M,K] * B[K,N].
//
// Used for every projection of the round: Q/K/V/O of the reference attention
// and Q/O of the motion cross-attention (PersonaLive write-up, "三条条件通路"),
// and the K/V projection of reference/anchor features into the KV bank.
#pragma once
#include <cuda.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace pl {

constexpr int kGemmBM = 128;       // rows per tile (one TMEM lane per row)
constexpr int kGemmBK = 64;        // K per stage: one 128-byte swizzle atom of fp16
constexpr int kGemmBN = 160;       // columns per tile (MMA N); divides 3C, 2C and C of every level
constexpr int kGemmMaxProblems = 16;

struct GemmProblem {
  CUtensorMap a;        // 2D {K, M}, box {64, 128}, 128B swizzle (K-major A)
  CUtensorMap b;        // 2D {N, K}, box {64, 64}, 128B swizzle (MN-major B)
  CUtensorMap c;        // 2D {N, M}, box {32, 32}: fp16 with 64-byte swizzle or
                        // fp32 (out_f32) with 128-byte swizzle; stored by TMA
  int out_f32;
  int softmax32;              // fp16 output, each 32-column group replaced by the
                              // softmax of its values taken as base-2 logits
  int M, N, K;
  int tiles_n;
  int tile_begin, tile_end;   // linear tile range [begin, end)
  const int32_t* pred;        // when non-null the problem runs only if *pred != 0
};

struct GemmParams {
  GemmProblem prob[kGemmMaxProblems];
  int n_problems;
  int total_tiles;
  uint32_t* status;           // device status word (may be null)
};

// Host helpers (gemm.cu).
int gemm_make_problem(GemmProblem* p, const void* a, int64_t lda, const void* b, int64_t ldb,
                      void* c, int64_t ldc, int M, int N, int K, const int32_t* pred,
                      bool out_f32 = false);
// Set kernel attributes once (call outside stream capture). 0 on success.
int gemm_init();
// Turn a problem's epilogue into the 32-column softmax (fp16 output, N a
// multiple of 32). 0 on success.
int gemm_set_softmax32(GemmProblem* p);
// Launch a grouped GEMM over params->prob[0..n_problems). Fills tile ranges.
int gemm_launch(GemmParams* params, cudaStream_t stream, int max_ctas);

}  // namespace pl
