// Small bandwidth-bound kernels around the contractions: time-embedding
// sinusoid and GEMVs, nearest 2x upsampling, stride-2 phase split, and the
// conv_in operand builder.
#include "common.cuh"
#include "kernels.cuh"

namespace sdk {

// Sinusoidal time embedding (tutorial page, sinusoidal embedding paragraph):
// [cos(t f_i) | sin(t f_i)], f_i = exp(-ln(10000) i / half), evaluated in FP64.
__global__ void sinusoid_kernel(float t, int half, float* out) {
  pdl_wait();
  pdl_trigger();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= half) return;
  const double f = exp(-9.210340371976184 * (double)i / (double)half);  // ln(10000)
  const double a = (double)t * f;
  out[i] = (float)cos(a);
  out[half + i] = (float)sin(a);
}

int launch_sinusoid(float t, int proj_dim, float* out, cudaStream_t st) {
  const int half = proj_dim / 2;
  return (int)launch_pdl(sinusoid_kernel, dim3((half + 127) / 128), dim3(128), 0, st, t, half, out);
}

// Grouped GEMV: one warp per output row, 16-byte weight loads, x staged in
// shared memory with the optional input SiLU applied once.
__global__ void gemv_kernel(const __grid_constant__ GemvBatch batch) {
  extern __shared__ float xs[];
  pdl_wait();
  pdl_trigger();
  for (int k = threadIdx.x; k < batch.K; k += blockDim.x) {
    const float v = batch.x[k];
    xs[k] = batch.silu_in ? silu_f(v) : v;
  }
  __syncthreads();
  const int warps = blockDim.x >> 5;
  int row = blockIdx.x * warps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  int j = 0;
  while (j < batch.njobs && row >= batch.job[j].rows) {
    row -= batch.job[j].rows;
    ++j;
  }
  if (j >= batch.njobs) return;
  const GemvJob& job = batch.job[j];
  const __nv_bfloat16* w = job.W + (size_t)row * batch.K;
  float acc = 0.f;
  for (int k = lane * 8; k < batch.K; k += 32 * 8) {
    const uint4 q = *reinterpret_cast<const uint4*>(w + k);
    acc += bf16lo(q.x) * xs[k] + bf16hi(q.x) * xs[k + 1] + bf16lo(q.y) * xs[k + 2] + bf16hi(q.y) * xs[k + 3] +
           bf16lo(q.z) * xs[k + 4] + bf16hi(q.z) * xs[k + 5] + bf16lo(q.w) * xs[k + 6] + bf16hi(q.w) * xs[k + 7];
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    if (job.b) acc += __bfloat162float(job.b[row]);
    const float r = batch.silu_out ? silu_f(acc) : acc;
    job.y[row] = batch.accum_out ? job.y[row] + r : r;
  }
}

int launch_gemv(const GemvBatch& batch, cudaStream_t st) {
  long rows = 0;
  for (int j = 0; j < batch.njobs; ++j) rows += batch.job[j].rows;
  const int warps = 8;
  const int blocks = (int)((rows + warps - 1) / warps);
  if (blocks == 0) return 0;
  return (int)launch_pdl(gemv_kernel, dim3(blocks), dim3(warps * 32), batch.K * sizeof(float), st, batch);
}

// SDXL added conditioning (tutorial page, SDXL conditioning paragraphs): the
// pooled text vector, then each size/crop scalar Fourier-encoded like the
// timestep, in FP32 for the first linear layer.
__global__ void add_embed_input_kernel(const __nv_bfloat16* __restrict__ text, int text_dim, AddIds ids, int n_ids,
                                       int dim, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int half = dim / 2;
  const int total = text_dim + n_ids * dim;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    if (i < text_dim) {
      out[i] = __bfloat162float(text[i]);
      continue;
    }
    const int j = (i - text_dim) / dim;
    const int k = (i - text_dim) % dim;
    const int fi = k < half ? k : k - half;
    const double f = exp(-9.210340371976184 * (double)fi / (double)half);  // ln(10000)
    const double a = (double)ids.v[j] * f;
    out[i] = (float)(k < half ? cos(a) : sin(a));
  }
}

int launch_add_embed_input(const __nv_bfloat16* text, int text_dim, const AddIds& ids, int n_ids, int dim,
                           float* out, cudaStream_t st) {
  const int total = text_dim + n_ids * dim;
  return (int)launch_pdl(add_embed_input_kernel, dim3((total + 255) / 256), dim3(256), 0, st, text, text_dim, ids,
                         n_ids, dim, out);
}

// VAE decoder input: y[p][o] = b[o] + sum_c W[o][c] * (z[p][c] * inv_scale), the
// latent divided by the scaling factor, then the 1x1 post-quantisation conv.
__global__ void vae_latent_in_kernel(const __nv_bfloat16* __restrict__ z, const __nv_bfloat16* __restrict__ w,
                                     const __nv_bfloat16* __restrict__ b, int lc, int64_t hw, float inv_scale,
                                     __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int64_t total = hw * lc;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t p = i / lc;
    const int o = (int)(i % lc);
    float acc = __bfloat162float(b[o]);
    for (int c = 0; c < lc; ++c)
      acc = fmaf(__bfloat162float(w[o * lc + c]), __bfloat162float(z[p * lc + c]) * inv_scale, acc);
    y[i] = __float2bfloat16_rn(acc);
  }
}

int launch_vae_latent_in(const __nv_bfloat16* z, const __nv_bfloat16* w, const __nv_bfloat16* b, int lc, int64_t hw,
                         float inv_scale, __nv_bfloat16* y, cudaStream_t st) {
  const int64_t total = hw * lc;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  return (int)launch_pdl(vae_latent_in_kernel, dim3(blocks), dim3(256), 0, st, z, w, b, lc, hw, inv_scale, y);
}

// Row softmax of FP32 scores: P[r][j] = exp(scale*(S[r][j] - max_j S[r][j])) / sum, as BF16.
// One CTA per row; the row is read once into shared memory.
__global__ void __launch_bounds__(256) softmax_rows_kernel(const float* __restrict__ S, int64_t ld_s, int n,
                                                           float scale_log2, __nv_bfloat16* __restrict__ P,
                                                           int64_t ld_p) {
  extern __shared__ float row[];
  __shared__ float red[8];
  pdl_wait();
  pdl_trigger();
  const float* src = S + (int64_t)blockIdx.x * ld_s;
  float mx = -INFINITY;
  for (int j = threadIdx.x * 4; j < n; j += blockDim.x * 4) {
    const float4 v = *reinterpret_cast<const float4*>(src + j);
    *reinterpret_cast<float4*>(row + j) = v;
    mx = fmaxf(fmaxf(mx, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
  }
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) red[wid] = mx;
  __syncthreads();
  mx = red[0];
  for (int k = 1; k < (int)(blockDim.x >> 5); ++k) mx = fmaxf(mx, red[k]);
  __syncthreads();
  const float m = mx * scale_log2;
  float sum = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float e = exp2f(fmaf(row[j], scale_log2, -m));
    row[j] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) red[wid] = sum;
  __syncthreads();
  float tot = 0.f;
  for (int k = 0; k < (int)(blockDim.x >> 5); ++k) tot += red[k];
  const float inv = 1.f / tot;
  __nv_bfloat16* dst = P + (int64_t)blockIdx.x * ld_p;
  for (int j = threadIdx.x * 8; j < n; j += blockDim.x * 8) {
    *reinterpret_cast<uint4*>(dst + j) =
        make_uint4(pack_bf16x2(row[j] * inv, row[j + 1] * inv), pack_bf16x2(row[j + 2] * inv, row[j + 3] * inv),
                   pack_bf16x2(row[j + 4] * inv, row[j + 5] * inv), pack_bf16x2(row[j + 6] * inv, row[j + 7] * inv));
  }
}

int launch_softmax_rows(const float* S, int64_t ld_s, int rows, int n, float scale, __nv_bfloat16* P, int64_t ld_p,
                        cudaStream_t st) {
  if (n % 8 || ld_s % 4 || ld_p % 8) return -1;
  const size_t smem = (size_t)n * sizeof(float);
  if (smem > 200 * 1024) return -1;
  static bool attr = false;  // benign race: identical value for every caller
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(softmax_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess) return (int)e;
    attr = true;
  }
  return (int)launch_pdl(softmax_rows_kernel, dim3(rows), dim3(256), smem, st, S, ld_s, n,
                         scale * 1.4426950408889634f, P, ld_p);
}

// dst[c][r] = src[r][c0 + c] for r < rows, c < cols (32 x 32 tiles through shared memory).
__global__ void transpose_kernel(const __nv_bfloat16* __restrict__ src, int64_t ld_src, int c0, int rows, int cols,
                                 __nv_bfloat16* __restrict__ dst, int64_t ld_dst) {
  __shared__ __nv_bfloat16 tile[32][33];
  pdl_wait();
  pdl_trigger();
  const int r0 = blockIdx.y * 32, cb = blockIdx.x * 32;
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int r = r0 + k, c = cb + threadIdx.x;
    if (r < rows && c < cols) tile[k][threadIdx.x] = src[(int64_t)r * ld_src + c0 + c];
  }
  __syncthreads();
  for (int k = threadIdx.y; k < 32; k += blockDim.y) {
    const int c = cb + k, r = r0 + threadIdx.x;
    if (r < rows && c < cols) dst[(int64_t)c * ld_dst + r] = tile[threadIdx.x][k];
  }
}

int launch_transpose(const __nv_bfloat16* src, int64_t ld_src, int c0, int rows, int cols, __nv_bfloat16* dst,
                     int64_t ld_dst, cudaStream_t st) {
  return (int)launch_pdl(transpose_kernel, dim3((cols + 31) / 32, (rows + 31) / 32), dim3(32, 8), 0, st, src, ld_src,
                         c0, rows, cols, dst, ld_dst);
}

// Nearest 2x (UpSample bullet): y[i][j] = x[i/2][j/2], one 16-byte vector per thread.
__global__ void upsample2x_kernel(const uint4* __restrict__ x, int H, int W, int V, uint4* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const size_t total = (size_t)4 * H * W * V;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int v = (int)(idx % V);
    const size_t p = idx / V;
    const int oj = (int)(p % (2 * W));
    const int oi = (int)(p / (2 * W));
    y[idx] = x[((size_t)(oi >> 1) * W + (oj >> 1)) * V + v];
  }
}

int launch_upsample2x(const __nv_bfloat16* x, int H, int W, int C, __nv_bfloat16* y, cudaStream_t st) {
  const int V = C / 8;
  const size_t total = (size_t)4 * H * W * V;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (int)launch_pdl(upsample2x_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4*>(x), H, W,
                         V, reinterpret_cast<uint4*>(y));
}

// Phase split: plane (a, b) holds the pixels (2i + a, 2j + b).
__global__ void phase_split_kernel(const uint4* __restrict__ x, int H, int W, int V, uint4* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int Ho = H / 2, Wo = W / 2;
  const size_t total = (size_t)H * W * V;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int v = (int)(idx % V);
    const size_t p = idx / V;
    const int xx = (int)(p % W);
    const int yy = (int)(p / W);
    const int plane = (yy & 1) * 2 + (xx & 1);
    y[(((size_t)plane * Ho + (yy >> 1)) * Wo + (xx >> 1)) * V + v] = x[idx];
  }
}

int launch_phase_split(const __nv_bfloat16* x, int H, int W, int C, __nv_bfloat16* y, cudaStream_t st) {
  const int V = C / 8;
  const size_t total = (size_t)H * W * V;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (int)launch_pdl(phase_split_kernel, dim3(blocks), dim3(256), 0, st, reinterpret_cast<const uint4*>(x), H, W,
                         V, reinterpret_cast<uint4*>(y));
}

// conv_in operand (small C_in): one thread per output element.
__global__ void conv_in_im2col_kernel(const __nv_bfloat16* __restrict__ s0, int c0, const __nv_bfloat16* __restrict__ s1,
                                      int c1, const __nv_bfloat16* __restrict__ s2, int c2, int H, int W, int Kp,
                                      __nv_bfloat16* __restrict__ y) {
  pdl_wait();
  pdl_trigger();
  const int Cin = c0 + c1 + c2;
  const size_t total = (size_t)H * W * Kp;
  for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
       idx += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(idx % Kp);
    const size_t p = idx / Kp;
    float v = 0.f;
    if (k < 9 * Cin) {
      const int tap = k / Cin;
      const int c = k % Cin;
      const int yy = (int)(p / W) + tap / 3 - 1;
      const int xx = (int)(p % W) + tap % 3 - 1;
      if (yy >= 0 && yy < H && xx >= 0 && xx < W) {
        const size_t q = (size_t)yy * W + xx;
        if (c < c0)
          v = __bfloat162float(s0[q * c0 + c]);
        else if (c < c0 + c1)
          v = __bfloat162float(s1[q * c1 + (c - c0)]);
        else
          v = __bfloat162float(s2[q * c2 + (c - c0 - c1)]);
      }
    }
    y[idx] = __float2bfloat16_rn(v);
  }
}

int launch_conv_in_im2col(const __nv_bfloat16* s0, int c0, const __nv_bfloat16* s1, int c1,
                          const __nv_bfloat16* s2, int c2, int H, int W, int Kp, __nv_bfloat16* y,
                          cudaStream_t st) {
  const size_t total = (size_t)H * W * Kp;
  int blocks = (int)((total + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  return (int)launch_pdl(conv_in_im2col_kernel, dim3(blocks), dim3(256), 0, st, s0, c0, s1, c1, s2, c2, H, W, Kp, y);
}

}  // namespace sdk
