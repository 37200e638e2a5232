// Launchers of the non-GEMM kernels. Each returns 0 or a cudaError_t value.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sdk {

// GroupNorm statistics accumulators: group g's fixed-point sum and sum of squares
// are words kGnAccStride*g and kGnAccStride*g + 1, so every group has a 128-byte
// line of its own (the atomics of all CTAs on one group do not queue behind
// those of the other groups).
constexpr int kGnAccStride = 16;

// GroupNorm (+SiLU) of the channel concatenation [x0 | x1] (x1 may be null with
// C1 = 0) into y. `acc` holds kGnAccStride*G zero-initialised words and `counter`
// one zero-initialised word used by this call only. When each CTA's share of the pixels fits in shared memory
// one kernel does both passes (statistics, grid barrier, normalisation; a
// barrier that times out raises ERR_MBAR_TIMEOUT in *err); otherwise a
// statistics kernel and an apply kernel run (counter / err may then be null).
int launch_groupnorm(const __nv_bfloat16* x0, int C0, const __nv_bfloat16* x1, int C1, int HW, int G, float eps,
                     const __nv_bfloat16* gamma, const __nv_bfloat16* beta, int silu, __nv_bfloat16* y,
                     unsigned long long* acc, unsigned int* counter, int num_sms, cudaStream_t st, int* err);
// Kernels launch_groupnorm enqueues for these sizes (1 or 2).
int groupnorm_plan_launches(int C, int HW, int num_sms);
// Time embedding: phi(t) sinusoid [proj_dim] into out (FP32).
int launch_sinusoid(float t, int proj_dim, float* out, cudaStream_t st);

// Grouped GEMV: for each job, y[r] = act_out(sum_k W[r][k] * act_in(x[k]) + b[r]),
// W BF16 [rows][K] row-major, x FP32 [K] shared by all jobs; with accum_out the
// result is added to y[r] instead of replacing it.
constexpr int kMaxGemvJobs = 32;
struct GemvJob {
  const __nv_bfloat16* W;
  const __nv_bfloat16* b;
  float* y;
  int32_t rows;
};
struct GemvBatch {
  int32_t njobs, K, silu_in, silu_out, accum_out;
  const float* x;
  GemvJob job[kMaxGemvJobs];
};
int launch_gemv(const GemvBatch& batch, cudaStream_t st);

// SDXL added-conditioning input: out = [text (BF16 -> FP32) | phi(ids[0]) | ... ],
// phi(v) = [cos(v f_i) | sin(v f_i)] of width dim, f_i = 10000^(-i/(dim/2)).
constexpr int kMaxAddIds = 8;
struct AddIds {
  float v[kMaxAddIds];
};
int launch_add_embed_input(const __nv_bfloat16* text, int text_dim, const AddIds& ids, int n_ids, int dim,
                           float* out, cudaStream_t st);

// VAE decoder input: y = 1x1 conv (W [lc][lc], b [lc]) of z * inv_scale, NHWC [hw][lc].
int launch_vae_latent_in(const __nv_bfloat16* z, const __nv_bfloat16* w, const __nv_bfloat16* b, int lc, int64_t hw,
                         float inv_scale, __nv_bfloat16* y, cudaStream_t st);
// Row softmax: P[r][:] = softmax(scale * S[r][:]) as BF16 for rows x n FP32 scores
// (n a multiple of 8, at most 51200). Returns -1 for unsupported sizes.
int launch_softmax_rows(const float* S, int64_t ld_s, int rows, int n, float scale, __nv_bfloat16* P, int64_t ld_p,
                        cudaStream_t st);
// dst[c][r] = src[r][c0 + c] (BF16), rows x cols.
int launch_transpose(const __nv_bfloat16* src, int64_t ld_src, int c0, int rows, int cols, __nv_bfloat16* dst,
                     int64_t ld_dst, cudaStream_t st);

// Nearest 2x upsample of NHWC [H, W, C] into [2H, 2W, C].
int launch_upsample2x(const __nv_bfloat16* x, int H, int W, int C, __nv_bfloat16* y, cudaStream_t st);

// Phase split for the stride-2 convolution: y[a*2+b][i][j][c] = x[2i+a][2j+b][c].
int launch_phase_split(const __nv_bfloat16* x, int H, int W, int C, __nv_bfloat16* y, cudaStream_t st);

// conv_in operand: y[p][k] for k = (ky*3 + kx)*Cin + c (0 beyond 9*Cin, up to Kp),
// reading input channel c from the source that holds it (up to 3 sources of
// widths c0/c1/c2 concatenated on channels), zero outside the image.
int launch_conv_in_im2col(const __nv_bfloat16* s0, int c0, const __nv_bfloat16* s1, int c1,
                          const __nv_bfloat16* s2, int c2, int H, int W, int Kp, __nv_bfloat16* y,
                          cudaStream_t st);

// Flash attention on tcgen05 (head_dim 64): O[i, h*64 + d] = softmax_j(Q_i.K_j / 8) V_j
// per head; Q rows come from a [q_rows, q_ld] matrix at column q_col + 64h, K and V
// from a [kv_rows, kv_ld] matrix at columns k_col + 64h and v_col + 64h. Where it
// pays, the key tiles of the (head, query tile) items are spread evenly over
// 2*num_sms CTAs; the pieces of split items go through `partial`
// (attention_partial_bytes(num_sms) bytes; null disables splitting) and are merged
// by a second kernel. attention_plan_launches gives the number of kernels (1 or 2).
size_t attention_partial_bytes(int num_sms);
int attention_plan_launches(int Nq, int Nk, int heads, int num_sms);
int launch_attention_tc(const __nv_bfloat16* qbase, int q_ld, int q_rows, int q_col, const __nv_bfloat16* kvbase,
                        int kv_ld, int kv_rows, int k_col, int v_col, __nv_bfloat16* O, int ldo, int Nq, int Nk,
                        int heads, float* partial, size_t partial_bytes, int num_sms, int* err, cudaStream_t st);

}  // namespace sdk
