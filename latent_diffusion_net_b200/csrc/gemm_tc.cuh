// Host-visible description of the tcgen05 implicit-GEMM used for every dense
// contraction of the denoiser: 3x3 convolutions (9 shifted K-segments over an
// NHWC activation), stride-2 convolutions (9 segments over 4 phase planes),
// 1x1 shortcut convolutions fused as extra K-segments, and token linears.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdk {

constexpr int kGemmMaxSeg = 12;
constexpr int kGemmMaxA = 4;
constexpr int kGemmMaxB = 2;

// GEMM_F32: the output (after the biases) is stored as FP32 to (float*)out with
// row stride ld_out elements; no residual, no split reduction.
enum GemmMode : int32_t { GEMM_PLAIN = 0, GEMM_GEGLU = 1, GEMM_F32 = 2 };

// One activation source: a BF16 NHWC tensor seen as [Z][H][W][C].
struct GemmASrc {
  const void* ptr;
  int32_t C, W, H, Z;
};

// One weight matrix: BF16 [rows][K] row-major (rows = output features).
struct GemmBSrc {
  const void* ptr;
  int32_t K, rows;
};

// K-segment: nkb blocks of 64 reduction elements read from A source `amap` at
// channel c0 with the output tile shifted by (dx, dy) on plane z, against B
// source `bmap` starting at reduction index bk0.
struct GemmSeg {
  int32_t amap, bmap;
  int32_t dx, dy, z;
  int32_t c0, bk0, nkb;
};

struct GemmEpi {
  const __nv_bfloat16* bias;      // [N] or null
  const __nv_bfloat16* bias2;     // [N] or null (second bias, e.g. a fused shortcut)
  const float* colvec;            // [N] FP32 or null (time-embedding projection)
  const __nv_bfloat16* residual;  // [M][ld_res] or null, added after the biases
  int32_t ld_res;
  __nv_bfloat16* out;             // [M][ld_out]
  int32_t ld_out;
  int32_t mode;                   // GemmMode
  int32_t f16_begin;              // > 0: output columns >= f16_begin are stored as FP16 (a multiple of 32)
  // Row statistics for a LayerNorm folded into the next GEMM. rowstat_out: each
  // output row's sum and sum of squares of the stored BF16 values are added into
  // rowstat_out[2*row .. 2*row+1] as 64-bit fixed point (scales 2^24 and 2^18);
  // the buffer must be zero before the launch. rowstat_in: the A operand is the
  // raw (not normalised) input x whose row sums are there; the epilogue then
  // forms rstd*(acc - mean*colscale[n]) + colvec[n] with mean and rstd over
  // ln_cols values and ln_eps (a LayerNorm with gamma folded into B, colscale =
  // row sums of that B, colvec = B times beta plus bias).
  unsigned long long* rowstat_out;
  const unsigned long long* rowstat_in;
  // Zeroed by this launch once every earlier kernel on the stream has finished
  // (the other row-statistics buffer, whose last reader ran before).
  unsigned long long* rowstat_clear;
  int64_t rowstat_clear_elems;
  const float* colscale;
  int32_t ln_cols;
  float ln_eps;
};

constexpr double kRowSumScale = 16777216.0;  // 2^24
constexpr double kRowSqScale = 262144.0;     // 2^18

// A full problem: output grid Ho x Wo (M = Ho*Wo rows), N output features.
// When its cost model says it pays and an FP32 split-K buffer is given, the
// planner splits the reduction into K ranges (separate work units of the
// persistent kernel) and a second kernel adds the partial products in a fixed
// order and applies the epilogue.
struct GemmProblem {
  int32_t Ho, Wo, N;
  int32_t na, nb, nseg;
  GemmASrc a[kGemmMaxA];
  GemmBSrc b[kGemmMaxB];
  GemmSeg seg[kGemmMaxSeg];
  GemmEpi epi;
  int* err;
  int32_t force_bn;      // 0 = heuristic
  int32_t force_splits;  // 0 = heuristic, 1 = no split
  float* splitk_ws;      // FP32 partials [splits][Ho*Wo][N], or null
  size_t splitk_ws_bytes;
  // > 0 (tests only): one thread of every CTA first waits on a barrier nothing
  // completes, for at most hold_spins polls; the wait gives up and the CTA
  // skips all its work (see sd_debug_inject_timeout)
  int32_t hold_spins;
};

// Number of kernels gemm_tc_launch will enqueue for p (1, or 2 with split-K).
int gemm_tc_plan_launches(const GemmProblem& p);

// Launch on `stream`. Returns 0 on success, a cudaError_t value otherwise
// (or -1 for an unsupported shape).
int gemm_tc_launch(const GemmProblem& p, cudaStream_t stream);

// Tensor-map encoder from the driver (resolved once, no -lcuda needed).
bool tmap_encode_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                    uint32_t box_outer);
bool tmap_encode_4d(CUtensorMap* m, const void* ptr, const uint64_t dims[4], uint32_t box_w, uint32_t box_h);

}  // namespace sdk
