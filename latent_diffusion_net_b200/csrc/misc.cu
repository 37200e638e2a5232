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
