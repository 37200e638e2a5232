// Flash attention, head_dim 64, for self-attention over the H*W image tokens
// and cross-attention over the 77 context rows (SD1.5 anatomy page, section
// 3.4: Softmax(Q K^T / sqrt(d)) V; Transformer2DModel panel of the SD2.1 page,
// section 4: Q = K = V = image tokens, and K = V = context).
//
// One CTA = 64 queries of one head, 4 warps x 16 query rows. K/V tiles of 64
// keys are double-buffered in shared memory with cp.async (zero-filled past the
// last key, masked to -inf in the scores). Scores and the output accumulate in
// registers through mma.sync m16n8k16 (BF16 in, FP32 accumulate); the softmax
// is online in the exp2 domain with per-row running max and sum. S and P never
// touch global memory.
#include "common.cuh"
#include "kernels.cuh"

namespace sdk {

namespace {

constexpr int kQT = 64;  // queries per CTA
constexpr int kKT = 64;  // keys per tile
constexpr int kHD = 64;  // head dim

// Shared tile [64 rows][64 bf16] with the 16-byte chunks of row r XOR-swizzled by (r & 7).
__device__ __forceinline__ uint32_t swz(int r, int chunk) { return (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4)); }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Load a [64 x 64] tile (rows row0.., columns col0..col0+63 of a row-major
// matrix with leading dimension ld) into swizzled shared memory; rows >= nrows
// are zero-filled.
__device__ __forceinline__ void load_tile(uint32_t sbase, const __nv_bfloat16* g, int ld, int row0, int nrows) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int idx = threadIdx.x + i * 128;  // 512 chunks of 16 bytes
    const int r = idx >> 3;
    const int ch = idx & 7;
    const int gr = row0 + r;
    const bool valid = gr < nrows;
    const __nv_bfloat16* src = g + (size_t)(valid ? gr : 0) * ld + ch * 8;
    cp_async16(sbase + swz(r, ch), src, valid);
  }
}

}  // namespace

__global__ void __launch_bounds__(128) attention_kernel(const __nv_bfloat16* __restrict__ Q, int ldq,
                                                        const __nv_bfloat16* __restrict__ K, int ldk,
                                                        const __nv_bfloat16* __restrict__ V, int ldv,
                                                        __nv_bfloat16* __restrict__ O, int ldo, int Nq, int Nk,
                                                        float scale_log2) {
  __shared__ __align__(128) uint8_t smem[(kQT + 4 * kKT) * kHD * 2];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK0 = sQ + kQT * kHD * 2;
  const uint32_t sV0 = sK0 + 2 * kKT * kHD * 2;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int q0 = blockIdx.x * kQT;
  const int h = blockIdx.y;
  const __nv_bfloat16* Qh = Q + h * kHD;
  const __nv_bfloat16* Kh = K + h * kHD;
  const __nv_bfloat16* Vh = V + h * kHD;

  const int ntiles = (Nk + kKT - 1) / kKT;
  load_tile(sQ, Qh, ldq, q0, Nq);
  load_tile(sK0, Kh, ldk, 0, Nk);
  load_tile(sV0, Vh, ldv, 0, Nk);
  cp_async_commit();

  uint32_t qf[4][4];  // A fragments of this warp's 16 query rows, 4 k-steps of 16
  float oacc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_r[2] = {-INFINITY, -INFINITY};
  float l_r[2] = {0.f, 0.f};

  for (int j = 0; j < ntiles; ++j) {
    const int buf = j & 1;
    if (j + 1 < ntiles) {
      const uint32_t off = (uint32_t)((buf ^ 1) * kKT * kHD * 2);
      load_tile(sK0 + off, Kh, ldk, (j + 1) * kKT, Nk);
      load_tile(sV0 + off, Vh, ldv, (j + 1) * kKT, Nk);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (j == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int m = lane >> 3;
        const int r = warp * 16 + (m & 1) * 8 + (lane & 7);
        const int ch = kk * 2 + (m >> 1);
        ldsm_x4(sQ + swz(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    const uint32_t sK = sK0 + buf * kKT * kHD * 2;
    const uint32_t sV = sV0 + buf * kKT * kHD * 2;

    // S = Q K^T for 16 rows x 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {  // pairs of n-tiles (16 keys)
        const int m = lane >> 3;
        const int r = np * 16 + (m >> 1) * 8 + (lane & 7);
        const int ch = kk * 2 + (m & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz(r, ch), b0, b1, b2, b3);
        mma16816(s[2 * np], qf[kk], b0, b1);
        mma16816(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    // mask keys past the end
    const int kbase = j * kKT;
    if (kbase + kKT > Nk) {
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        const int key = kbase + n * 8 + (lane & 3) * 2;
        if (key >= Nk) s[n][0] = s[n][2] = -INFINITY;
        if (key + 1 >= Nk) s[n][1] = s[n][3] = -INFINITY;
      }
    }
    // online softmax: rows g (values 0,1) and g+8 (values 2,3)
    float mx[2] = {m_r[0], m_r[1]};
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      mx[0] = fmaxf(mx[0], fmaxf(s[n][0], s[n][1]));
      mx[1] = fmaxf(mx[1], fmaxf(s[n][2], s[n][3]));
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 1));
      mx[i] = fmaxf(mx[i], __shfl_xor_sync(0xffffffffu, mx[i], 2));
    }
    float alpha[2], mb[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      mb[i] = (mx[i] == -INFINITY) ? 0.f : mx[i] * scale_log2;
      alpha[i] = exp2f(m_r[i] * scale_log2 - mb[i]);
      m_r[i] = mx[i];
      l_r[i] *= alpha[i];
    }
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      oacc[n][0] *= alpha[0];
      oacc[n][1] *= alpha[0];
      oacc[n][2] *= alpha[1];
      oacc[n][3] *= alpha[1];
    }
    uint32_t pf[4][4];  // P as A fragments: 4 k-steps of 16 keys
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float p0 = exp2f(fmaf(s[n][0], scale_log2, -mb[0]));
      const float p1 = exp2f(fmaf(s[n][1], scale_log2, -mb[0]));
      const float p2 = exp2f(fmaf(s[n][2], scale_log2, -mb[1]));
      const float p3 = exp2f(fmaf(s[n][3], scale_log2, -mb[1]));
      l_r[0] += p0 + p1;
      l_r[1] += p2 + p3;
      const int kk = n >> 1;
      if ((n & 1) == 0) {
        pf[kk][0] = pack_bf16x2(p0, p1);
        pf[kk][1] = pack_bf16x2(p2, p3);
      } else {
        pf[kk][2] = pack_bf16x2(p0, p1);
        pf[kk][3] = pack_bf16x2(p2, p3);
      }
    }
    // O += P V : k = keys (4 steps of 16), n = head dims (8 tiles of 8)
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {  // pairs of dim tiles
        const int m = lane >> 3;
        const int r = kk * 16 + (m & 1) * 8 + (lane & 7);
        const int ch = dp * 2 + (m >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sV + swz(r, ch), b0, b1, b2, b3);
        mma16816(oacc[2 * dp], pf[kk], b0, b1);
        mma16816(oacc[2 * dp + 1], pf[kk], b2, b3);
      }
    }
    __syncthreads();
  }

  // finalise: divide by the row sums (reduced over the 4 threads of a row)
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 1);
    l_r[i] += __shfl_xor_sync(0xffffffffu, l_r[i], 2);
  }
  const float inv0 = l_r[0] > 0.f ? 1.f / l_r[0] : 0.f;
  const float inv1 = l_r[1] > 0.f ? 1.f / l_r[1] : 0.f;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int row0 = q0 + warp * 16 + g;
  const int row1 = row0 + 8;
  __nv_bfloat16* Oh = O + h * kHD;
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    const int col = n * 8 + 2 * t;
    if (row0 < Nq)
      *reinterpret_cast<uint32_t*>(Oh + (size_t)row0 * ldo + col) = pack_bf16x2(oacc[n][0] * inv0, oacc[n][1] * inv0);
    if (row1 < Nq)
      *reinterpret_cast<uint32_t*>(Oh + (size_t)row1 * ldo + col) = pack_bf16x2(oacc[n][2] * inv1, oacc[n][3] * inv1);
  }
}

int launch_attention(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K, int ldk, const __nv_bfloat16* V,
                     int ldv, __nv_bfloat16* O, int ldo, int Nq, int Nk, int heads, cudaStream_t st) {
  const float scale_log2 = 0.125f * 1.4426950408889634f;  // 1/sqrt(64) * log2(e)
  dim3 grid((Nq + kQT - 1) / kQT, heads);
  attention_kernel<<<grid, 128, 0, st>>>(Q, ldq, K, ldk, V, ldv, O, ldo, Nq, Nk, scale_log2);
  return (int)cudaGetLastError();
}

}  // namespace sdk
