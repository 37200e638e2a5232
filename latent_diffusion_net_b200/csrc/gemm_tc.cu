// tcgen05 implicit GEMM for sm_100a.
//
// D[M, N] = sum over K-segments of A_seg[M, 64*nkb] * B_seg[N, 64*nkb]^T, then
// epilogue: + bias + bias2 + colvec, + residual, BF16 store (or GEGLU pairs).
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads of A (4-D box of a
// BHxBW pixel rectangle x 64 channels, zero-filled outside the image, which is
// exactly the zero padding of a 3x3 convolution) and B (64 x BN weight tile);
// warp 1 owns the TMEM accumulator and lane 0 issues tcgen05.mma (M=128, N=BN,
// K=16, BF16 in, FP32 accumulate); warps 2..5 are the epilogue, one TMEM lane
// quarter each (warp w reads lanes 32*(w%4) .. +31).
#include "common.cuh"
#include "gemm_tc.cuh"

#include <mutex>

namespace sdk {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB

struct __align__(64) GemmMaps {
  CUtensorMap a[kGemmMaxA];
  CUtensorMap b[kGemmMaxB];
};

struct GemmArgs {
  int32_t Ho, Wo, BH, BW, tiles_x, N;
  int32_t nseg, total_kb;
  int32_t kb_per_split;  // k-blocks per blockIdx.z (== total_kb without split-K)
  GemmSeg seg[kGemmMaxSeg];
  GemmEpi epi;
  float* partial;  // split-K: FP32 [gridDim.z][Ho*Wo][N]; null otherwise
  int* err;
};

template <int BN>
struct TmemCols {
  static constexpr uint32_t value = BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
};

__device__ __forceinline__ float gelu_erf(float g) { return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)); }

template <int BN, int STAGES>
__global__ void __launch_bounds__(192, 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args) {
  constexpr int kBTileBytes = BN * kBK * 2;
  constexpr int kStageBytes = kATileBytes + kBTileBytes;
  constexpr uint32_t kTmemCols = TmemCols<BN>::value;
  constexpr uint32_t kIdesc = umma_idesc_bf16(kBM, BN);
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "epilogue works in 32-column chunks");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* accum_bar = empty_bar + STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_col = reinterpret_cast<float*>(tmem_slot + 4);  // [BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int mt = blockIdx.x;
  const int n0 = blockIdx.y * BN;
  const int tile_y0 = (mt / args.tiles_x) * args.BH;
  const int tile_x0 = (mt % args.tiles_x) * args.BW;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // everything above touched only shared memory and TMEM: wait for the previous kernel here
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < kGemmMaxA; ++i) tma_prefetch_desc(&maps.a[i]);
      tma_prefetch_desc(&maps.b[0]);
      tma_prefetch_desc(&maps.b[1]);
      const int kb_lo = blockIdx.z * args.kb_per_split;
      const int kb_hi = min(args.total_kb, kb_lo + args.kb_per_split);
      int g = 0;  // position in the whole reduction
      bool ok = true;
      for (int si = 0; si < args.nseg && ok && g < kb_hi; ++si) {
        const GemmSeg sg = args.seg[si];
        for (int j = 0; j < sg.nkb; ++j, ++g) {
          if (g < kb_lo) continue;
          if (g >= kb_hi) break;
          const int kb = g - kb_lo;
          const int s = kb % STAGES;
          const int it = kb / STAGES;
          if (kb >= STAGES && !mbar_wait(&empty_bar[s], (it - 1) & 1, abort_flag, args.err)) {
            ok = false;
            break;
          }
          uint8_t* a_dst = smem + s * kStageBytes;
          uint8_t* b_dst = a_dst + kATileBytes;
          mbar_arrive_expect_tx(&full_bar[s], kStageBytes);
          tma_load_4d(a_dst, &maps.a[sg.amap], &full_bar[s], sg.c0 + j * kBK, tile_x0 + sg.dx, tile_y0 + sg.dy,
                      sg.z);
          tma_load_2d(b_dst, &maps.b[sg.bmap], &full_bar[s], sg.bk0 + j * kBK, n0);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      const int kb_lo = blockIdx.z * args.kb_per_split;
      const int nkb = min(args.total_kb, kb_lo + args.kb_per_split) - kb_lo;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % STAGES;
        const int it = kb / STAGES;
        if (!mbar_wait(&full_bar[s], it & 1, abort_flag, args.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * kStageBytes);
        const uint32_t b_addr = a_addr + kATileBytes;
        const uint64_t adesc = umma_desc_k_sw128(a_addr);
        const uint64_t bdesc = umma_desc_k_sw128(b_addr);
#pragma unroll
        for (int k = 0; k < kBK / 16; ++k) {
          // +32 bytes along K inside the 128-byte swizzle row = +2 in the encoded address
          umma_bf16(tmem_base, adesc + 2 * k, bdesc + 2 * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
        }
        umma_commit(&empty_bar[s]);
      }
      if (ok) umma_commit(accum_bar);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;  // 0..127
    for (int c = et; c < BN; c += 128) {
      const int n = n0 + c;
      float v = 0.f;
      if (n < args.N && !args.partial) {
        if (args.epi.bias) v += __bfloat162float(args.epi.bias[n]);
        if (args.epi.bias2) v += __bfloat162float(args.epi.bias2[n]);
        if (args.epi.colvec) v += args.epi.colvec[n];
      }
      epi_col[c] = v;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const bool have = mbar_wait(accum_bar, 0, abort_flag, args.err);
    tc_fence_after();
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int oy = tile_y0 + row / args.BW;
    const int ox = tile_x0 + row % args.BW;
    const bool valid = have && oy < args.Ho && ox < args.Wo;
    const long grow = (long)oy * args.Wo + ox;
#pragma unroll 1
    for (int cc = 0; cc < BN / 32; ++cc) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) + cc * 32, r);
      tmem_ld_wait();
      if (!valid) continue;
      const int nb = n0 + cc * 32;
      if (nb >= args.N) continue;
      float v[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]) + epi_col[cc * 32 + j];
      const bool full = (nb + 32 <= args.N);
      if (args.partial) {
        float* dst = args.partial + ((size_t)blockIdx.z * args.Ho * args.Wo + grow) * args.N + nb;
        if (full) {
          float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
          for (int u = 0; u < 8; ++u) d4[u] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nb + j < args.N) dst[j] = v[j];
        }
        continue;
      }
      if (args.epi.mode == GEMM_GEGLU) {
        // columns (2j, 2j+1) hold (value_j, gate_j); output column (nb/2 + j)
        uint32_t o[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float a0 = v[4 * j] * gelu_erf(v[4 * j + 1]);
          const float a1 = v[4 * j + 2] * gelu_erf(v[4 * j + 3]);
          o[j] = pack_bf16x2(a0, a1);
        }
        __nv_bfloat16* dst = args.epi.out + grow * args.epi.ld_out + (nb >> 1);
        if (full) {
          uint4* d4 = reinterpret_cast<uint4*>(dst);
          d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
          d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            if (nb + 2 * j < args.N) {
              const uint32_t w = o[j >> 1];
              dst[j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (w >> 16) : (w & 0xFFFF)));
            }
          }
        }
        continue;
      }
      if (args.epi.residual) {
        const __nv_bfloat16* rs = args.epi.residual + grow * args.epi.ld_res + nb;
        if (full) {
          const uint4* r4 = reinterpret_cast<const uint4*>(rs);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 w = r4[u];
            v[8 * u + 0] += bf16lo(w.x);
            v[8 * u + 1] += bf16hi(w.x);
            v[8 * u + 2] += bf16lo(w.y);
            v[8 * u + 3] += bf16hi(w.y);
            v[8 * u + 4] += bf16lo(w.z);
            v[8 * u + 5] += bf16hi(w.z);
            v[8 * u + 6] += bf16lo(w.w);
            v[8 * u + 7] += bf16hi(w.w);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (nb + j < args.N) v[j] += __bfloat162float(rs[j]);
        }
      }
      __nv_bfloat16* dst = args.epi.out + grow * args.epi.ld_out + nb;
      if (full && args.epi.f16_begin > 0 && nb >= args.epi.f16_begin) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          d4[u] = make_uint4(pack_f16x2(v[8 * u + 0], v[8 * u + 1]), pack_f16x2(v[8 * u + 2], v[8 * u + 3]),
                             pack_f16x2(v[8 * u + 4], v[8 * u + 5]), pack_f16x2(v[8 * u + 6], v[8 * u + 7]));
        }
      } else if (full) {
        uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          d4[u] = make_uint4(pack_bf16x2(v[8 * u + 0], v[8 * u + 1]), pack_bf16x2(v[8 * u + 2], v[8 * u + 3]),
                             pack_bf16x2(v[8 * u + 4], v[8 * u + 5]), pack_bf16x2(v[8 * u + 6], v[8 * u + 7]));
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (nb + j < args.N) dst[j] = __float2bfloat16_rn(v[j]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// Split-K reduction: out = epilogue(sum over splits of partial), 8 columns per
// thread, splits added in index order (deterministic).
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N, GemmEpi epi) {
  pdl_wait();
  pdl_trigger();
  const int V = N / 8;
  const size_t total = (size_t)M * V;
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int row = (int)(i / V);
    const int c = (int)(i % V) * 8;
    float v[8];
    const float4* p0 = reinterpret_cast<const float4*>(partial + (size_t)row * N + c);
    float4 a = p0[0], b = p0[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    for (int z = 1; z < splits; ++z) {
      const float4* pz = reinterpret_cast<const float4*>(partial + ((size_t)z * M + row) * N + c);
      a = pz[0];
      b = pz[1];
      v[0] += a.x; v[1] += a.y; v[2] += a.z; v[3] += a.w; v[4] += b.x; v[5] += b.y; v[6] += b.z; v[7] += b.w;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float add = 0.f;
      if (epi.bias) add += __bfloat162float(epi.bias[c + j]);
      if (epi.bias2) add += __bfloat162float(epi.bias2[c + j]);
      if (epi.colvec) add += epi.colvec[c + j];
      v[j] += add;
    }
    if (epi.mode == GEMM_GEGLU) {
      const uint32_t o0 = pack_bf16x2(v[0] * gelu_erf(v[1]), v[2] * gelu_erf(v[3]));
      const uint32_t o1 = pack_bf16x2(v[4] * gelu_erf(v[5]), v[6] * gelu_erf(v[7]));
      *reinterpret_cast<uint2*>(epi.out + (size_t)row * epi.ld_out + c / 2) = make_uint2(o0, o1);
      continue;
    }
    if (epi.residual) {
      const uint4 r = *reinterpret_cast<const uint4*>(epi.residual + (size_t)row * epi.ld_res + c);
      v[0] += bf16lo(r.x); v[1] += bf16hi(r.x); v[2] += bf16lo(r.y); v[3] += bf16hi(r.y);
      v[4] += bf16lo(r.z); v[5] += bf16hi(r.z); v[6] += bf16lo(r.w); v[7] += bf16hi(r.w);
    }
    if (epi.f16_begin > 0 && c >= epi.f16_begin)
      *reinterpret_cast<uint4*>(epi.out + (size_t)row * epi.ld_out + c) =
          make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]), pack_f16x2(v[6], v[7]));
    else
      *reinterpret_cast<uint4*>(epi.out + (size_t)row * epi.ld_out + c) =
          make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
}

// ------------------------------------------------------------------ host side

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

bool tmap_encode_2d(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_inner,
                    uint32_t box_outer) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tmap_encode_4d(CUtensorMap* m, const void* ptr, const uint64_t d[4], uint32_t box_w, uint32_t box_h) {
  EncodeTiledFn enc = get_encoder();
  if (!enc) return false;
  cuuint64_t dims[4] = {d[0], d[1], d[2], d[3]};
  cuuint64_t strides[3] = {d[0] * 2, d[0] * d[1] * 2, d[0] * d[1] * d[2] * 2};
  cuuint32_t box[4] = {64, box_w, box_h, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES>
static int launch_bn(const GemmMaps& maps, const GemmArgs& args, int tiles_m, int tiles_n, int splits,
                     cudaStream_t st) {
  constexpr int kStageBytes = kATileBytes + BN * kBK * 2;
  constexpr size_t smem = 1024 + (size_t)STAGES * kStageBytes + 256 + BN * 4;
  static bool attr_set = false;  // benign race: the attribute value is identical for every caller
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return (int)e;
    attr_set = true;
  }
  return (int)launch_pdl(gemm_tc_kernel<BN, STAGES>, dim3(tiles_m, tiles_n, splits), dim3(192), smem, st, maps, args);
}

static void choose_tile_rect(int Ho, int Wo, int* BH, int* BW) {
  if (Ho == 1) {
    *BH = 1;
    *BW = 128;
    return;
  }
  int best = -1, bw_best = 16;
  const int cands[] = {16, 32, 8, 64, 4, 128};
  for (int bw : cands) {
    int bh = 128 / bw;
    int tiles = ((Wo + bw - 1) / bw) * ((Ho + bh - 1) / bh);
    if (best < 0 || tiles < best) {
      best = tiles;
      bw_best = bw;
    }
  }
  *BW = bw_best;
  *BH = 128 / bw_best;
}

static int choose_bn(int N, int tiles_m, int num_sms) {
  if (N <= 32) return 32;
  const int cands[] = {256, 192, 160, 128, 64};
  for (int bn : cands) {
    if (N % bn) continue;
    if ((long)tiles_m * (N / bn) >= (long)num_sms * 9 / 10) return bn;
  }
  if (N % 64 == 0) return 64;
  return 0;
}

struct GemmPlan {
  int BH, BW, tiles_x, tiles_m, bn, tiles_n, splits, kb_per_split, total_kb;
};

static int sm_count() {
  static int num_sms = 0;
  if (num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (num_sms <= 0) num_sms = 148;
  }
  return num_sms;
}

// Tile shape, N tile and split-K factor for a problem.
static bool plan_gemm(const GemmProblem& p, GemmPlan* g) {
  const int sms = sm_count();
  choose_tile_rect(p.Ho, p.Wo, &g->BH, &g->BW);
  g->tiles_x = (p.Wo + g->BW - 1) / g->BW;
  g->tiles_m = g->tiles_x * ((p.Ho + g->BH - 1) / g->BH);
  g->total_kb = 0;
  for (int i = 0; i < p.nseg; ++i) g->total_kb += p.seg[i].nkb;
  g->bn = p.force_bn ? p.force_bn : choose_bn(p.N, g->tiles_m, sms);
  if (g->bn == 0 || g->total_kb <= 0) return false;
  g->splits = 1;
  // under-filled grid with a long reduction: a 128-wide N tile and split-K
  const bool small = (long)g->tiles_m * (p.N / 64 > 0 ? p.N / 64 : 1) < sms && g->total_kb >= 16 && p.N % 128 == 0;
  if (p.force_splits > 0) {
    g->splits = p.force_splits;
  } else if (small && p.splitk_ws && !p.force_bn) {
    g->bn = 128;
    const int ctas = g->tiles_m * (p.N / 128);
    int sp = (sms + ctas - 1) / ctas;
    if (sp > g->total_kb / 4) sp = g->total_kb / 4;
    if (sp > 16) sp = 16;
    const size_t per = (size_t)p.Ho * p.Wo * p.N * sizeof(float);
    while (sp > 1 && per * sp > p.splitk_ws_bytes) --sp;
    g->splits = sp < 1 ? 1 : sp;
  }
  g->tiles_n = (p.N + g->bn - 1) / g->bn;
  g->kb_per_split = (g->total_kb + g->splits - 1) / g->splits;
  g->splits = (g->total_kb + g->kb_per_split - 1) / g->kb_per_split;  // no empty split
  if (g->splits > 1 && (!p.splitk_ws || (size_t)p.Ho * p.Wo * p.N * sizeof(float) * g->splits > p.splitk_ws_bytes ||
                        p.N % 8))
    return false;
  return true;
}

int gemm_tc_plan_launches(const GemmProblem& p) {
  GemmPlan g;
  if (!plan_gemm(p, &g)) return 1;
  return g.splits > 1 ? 2 : 1;
}

int gemm_tc_launch(const GemmProblem& p, cudaStream_t stream) {
  if (p.nseg <= 0 || p.nseg > kGemmMaxSeg || p.na <= 0 || p.na > kGemmMaxA || p.nb <= 0 || p.nb > kGemmMaxB)
    return -1;
  GemmPlan g;
  if (!plan_gemm(p, &g)) return -1;
  GemmArgs args{};
  args.Ho = p.Ho;
  args.Wo = p.Wo;
  args.BH = g.BH;
  args.BW = g.BW;
  args.tiles_x = g.tiles_x;
  args.N = p.N;
  args.nseg = p.nseg;
  for (int i = 0; i < p.nseg; ++i) args.seg[i] = p.seg[i];
  args.total_kb = g.total_kb;
  args.kb_per_split = g.kb_per_split;
  args.epi = p.epi;
  args.partial = g.splits > 1 ? p.splitk_ws : nullptr;
  args.err = p.err;
  const int bn = g.bn;
  const int tiles_m = g.tiles_m;
  const int tiles_n = g.tiles_n;
  const int splits = g.splits;

  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int i = 0; i < kGemmMaxA; ++i) {
    const GemmASrc& a = p.a[i < p.na ? i : 0];
    uint64_t d[4] = {(uint64_t)a.C, (uint64_t)a.W, (uint64_t)a.H, (uint64_t)a.Z};
    if (!tmap_encode_4d(&maps.a[i], a.ptr, d, args.BW, args.BH)) return -2;
  }
  for (int i = 0; i < kGemmMaxB; ++i) {
    const GemmBSrc& b = p.b[i < p.nb ? i : 0];
    if (!tmap_encode_2d(&maps.b[i], b.ptr, (uint64_t)b.K, (uint64_t)b.rows, 64, (uint32_t)bn)) return -2;
  }
  int e;
  switch (bn) {
    case 32: e = launch_bn<32, 6>(maps, args, tiles_m, tiles_n, splits, stream); break;
    case 64: e = launch_bn<64, 4>(maps, args, tiles_m, tiles_n, splits, stream); break;
    case 128: e = launch_bn<128, 3>(maps, args, tiles_m, tiles_n, splits, stream); break;
    case 160: e = launch_bn<160, 3>(maps, args, tiles_m, tiles_n, splits, stream); break;
    case 192: e = launch_bn<192, 4>(maps, args, tiles_m, tiles_n, splits, stream); break;
    case 256: e = launch_bn<256, 4>(maps, args, tiles_m, tiles_n, splits, stream); break;
    default: return -1;
  }
  if (e != 0 || splits <= 1) return e;
  const int M = p.Ho * p.Wo;
  const size_t vecs = (size_t)M * (p.N / 8);
  int blocks = (int)((vecs + 255) / 256);
  if (blocks > sm_count() * 8) blocks = sm_count() * 8;
  return (int)launch_pdl(splitk_reduce_kernel, dim3(blocks), dim3(256), 0, stream, (const float*)p.splitk_ws, splits, M,
                         p.N, p.epi);
}

}  // namespace sdk
