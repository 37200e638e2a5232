// tcgen05 implicit GEMM for sm_100a.
//
// D[M, N] = sum over K-segments of A_seg[M, 64*nkb] * B_seg[N, 64*nkb]^T, then
// epilogue: + bias + bias2 + colvec, + residual, BF16 store (or GEGLU pairs),
// or FP32 partial sums for a split reduction.
//
// A operand: a 4-D TMA box of a BHxBW pixel rectangle x 64 channels, zero-
// filled outside the image, which is exactly the zero padding of a 3x3
// convolution; each 3x3 tap is one K-segment with the box shifted by (dx, dy).
// B operand: 64-wide K slices of the [N][K] weight matrix.
#include "common.cuh"
#include "gemm_tc.cuh"

#include <algorithm>
#include <mutex>

namespace sdk {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kATileBytes = kBM * kBK * 2;  // 16 KB
constexpr int kEpiThreads = 256;              // 8 epilogue warps, two per TMEM lane quarter
constexpr int kGemmThreads = 64 + kEpiThreads;

constexpr int kMaxStages = 12;
constexpr int kSmemLimit = 232448;  // dynamic shared memory per CTA on sm_100
constexpr int kSmemFixed = 1024 + 256 + 4096;  // alignment slack, barriers, per-column terms (2 x [2][256])

struct __align__(64) GemmMaps {
  CUtensorMap a[kGemmMaxA];   // BH x BW pixel boxes
  CUtensorMap at[kGemmMaxA];  // (BH + 2) x BW boxes of the folded 3-tap segments
  CUtensorMap b[kGemmMaxB];
};

// A pipeline stage carries at least 8 MMAs (the stage handshake costs about
// as much as 4 of them):
// taps == 1: `per` (1 or 2) consecutive 64-channel blocks, each a BH x BW box
//   shifted by (dx, dy) against its B slice at bk0 + 64*j;
// taps == 3: the three vertically adjacent taps (dy = -1, 0, +1) of one column
//   dx of a 3x3 kernel share one (BH + 2) x BW box of one channel block; tap t
//   reads rows [t*BW, t*BW + 128) of it (BW is a multiple of 8, so every view
//   starts on a 1024-byte swizzle atom) against the B slice at bk0 + t*bstep.
struct KSeg {
  int32_t amap, bmap, dx, dy, z, c0, bk0, nkb, taps, bstep, per;
};
__host__ __device__ inline int kseg_stages(const KSeg& k) { return (k.nkb + k.per - 1) / k.per; }

struct GemmArgs {
  int32_t Ho, Wo, BH, BW, tiles_x, tiles_m, N;
  int32_t nseg, total_kb;  // total_kb: pipeline stages of one output tile
  int32_t kb_per_split, splits, tiles_n, units;
  int32_t stages, stage_bytes, a_bytes;  // ring depth, bytes per stage, A region of a stage
  KSeg seg[kGemmMaxSeg];
  GemmEpi epi;
  float* partial;  // split-K: FP32 [splits][Ho*Wo][N]; null otherwise
  int* err;
  int32_t hold_spins;  // tests only: see GemmProblem::hold_spins
};

__device__ __forceinline__ float gelu_erf(float g) { return 0.5f * g * (1.0f + erff(g * 0.70710678118654752f)); }

// ------------------------------------------------------------------ 2-SM helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA loads of a CTA pair: the data lands in this CTA's shared memory, the
// transaction bytes are counted on the barrier of the even CTA of the pair.
constexpr uint32_t kPeerBitMask = 0xFEFFFFFFu;
__device__ __forceinline__ void tma2_load_2d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma2_load_4d(void* dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2,
                                             int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
      "%5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar) & kPeerBitMask), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_2sm(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_2sm(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// D[tmem] (+)= A[smem of both CTAs] * B[smem of both CTAs]^T, M = 256, issued by the even CTA.
__device__ __forceinline__ void umma2_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` in both CTAs of the pair once the issued MMAs complete.
__device__ __forceinline__ void umma2_commit_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)0x3)
      : "memory");
}

// ------------------------------------------------------------------ the kernel
// A cluster of two CTAs (one per SM) computes 256 x BN output tiles with
// tcgen05.mma.cta_group::2: each CTA loads the 128 rows of A of its own
// 128-pixel tile and BN/2 rows of B; the even CTA issues the MMAs, which read
// both CTAs' shared memory and write each CTA's half of the accumulator into its
// own TMEM. The cluster walks a static list of work units (pair of M tiles, N
// tile, K split); accumulators are double-buffered in TMEM so the epilogue of
// one unit overlaps the main loop of the next.
// Roles (320 threads per CTA): warp 0 lane 0 TMA producer (both CTAs); warp 1
// owns TMEM, lane 0 of the even CTA issues MMAs; warps 2-9 epilogue (TMEM lane
// quarter warp % 4; warps 2-5 take the even 32-column chunks, 6-9 the odd ones).
template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ GemmMaps maps, const __grid_constant__ GemmArgs args) {
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "epilogue works in 32-column chunks");
  constexpr int kBHalf = BN / 2;
  constexpr int kBTileBytes = kBHalf * kBK * 2;
  constexpr uint32_t kTmemCols = 512;  // two accumulators of up to 256 columns
  constexpr uint32_t kIdesc = umma_idesc_bf16(256, BN);
  constexpr int kChunks = BN / 32;
  const int STAGES = args.stages;
  const int stage_bytes = args.stage_bytes;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + STAGES * stage_bytes);
  uint64_t* empty_bar = full_bar + STAGES;
  uint64_t* acc_full = empty_bar + STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;       // [2], used in the even CTA
  uint64_t* hold_bar = acc_empty + 2;       // never completed (timeout test)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(hold_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* epi_col = reinterpret_cast<float*>(smem + STAGES * stage_bytes + 256);  // [2][256] added terms
  float* epi_scl = epi_col + 512;                                                // [2][256] LayerNorm colscale

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int cluster_id = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_full[0], 1);
    mbar_init(&acc_full[1], 1);
    mbar_init(&acc_empty[0], 2);
    mbar_init(&acc_empty[1], 2);
    mbar_init(hold_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // the tensor maps are kernel parameters, not data of the previous kernel: fetch
    // them into the descriptor cache while that kernel is still running
    for (int i = 0; i < kGemmMaxA; ++i) {
      tma_prefetch_desc(&maps.a[i]);
      tma_prefetch_desc(&maps.at[i]);
    }
    tma_prefetch_desc(&maps.b[0]);
    tma_prefetch_desc(&maps.b[1]);
    // touch the parameters the producer and MMA loops read before their first
    // load and MMA, so that their constant-cache misses also fall before the wait
    int touch = args.units + args.splits + args.tiles_n + args.tiles_x + args.tiles_m + args.BH + args.BW +
                args.kb_per_split + args.total_kb + args.nseg + args.a_bytes;
#pragma unroll
    for (int i = 0; i < kGemmMaxSeg; ++i) touch += args.seg[i].amap + args.seg[i].per + args.seg[i].bstep;
    asm volatile("" ::"r"(touch));
  }
  if (warp == 1) tmem_alloc_2sm(tmem_slot, kTmemCols);
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above touched only shared memory and TMEM: wait for the previous
  // kernel here. The producer thread (warp 0, lane 0) waits later, just before
  // its first load, so that the setup of its first stage overlaps that kernel too.
  auto after_wait = [&]() {
    pdl_trigger();
    if (args.epi.rowstat_clear) {
      // every kernel before this one has finished: the buffer's last reader among them
      const int64_t n2 = args.epi.rowstat_clear_elems / 2;
      ulonglong2* z = reinterpret_cast<ulonglong2*>(args.epi.rowstat_clear);
      for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n2; i += (int64_t)gridDim.x * blockDim.x)
        z[i] = make_ulonglong2(0ull, 0ull);
    }
  };
  if (threadIdx.x != 0) {
    pdl_wait();
    after_wait();
  }
  if (args.hold_spins > 0) {
    // timeout test: nothing ever arrives on hold_bar, so this bounded wait gives
    // up, raises the error flag and sets abort_flag; every role below then
    // skips its work (no load is issued, so none is in flight at the teardown)
    if (threadIdx.x == 0) mbar_wait(hold_bar, 0, abort_flag, args.err, (uint32_t)args.hold_spins);
    __syncthreads();
  }

  if (warp == 0) {
    bool waited = false;
    if (lane == 0 && !*abort_flag) {
      const uint32_t tall_bytes = (uint32_t)((args.BH + 2) * args.BW * kBK * 2 + 3 * kBTileBytes);
      const uint32_t single_bytes = (uint32_t)(kATileBytes + kBTileBytes);
      uint32_t q = 0;        // stages issued by this CTA so far
      int s = 0;             // ring slot of stage q
      uint32_t ph = 0;       // ring pass parity of stage q
      bool ok = true;
      for (int u = cluster_id; u < args.units && ok; u += nclusters) {
        const int z = u % args.splits;
        const int rest = u / args.splits;
        const int nt = rest % args.tiles_n;
        const int mt = (rest / args.tiles_n) * 2 + (int)rank;
        const int tile_y0 = (mt / args.tiles_x) * args.BH;  // past the image for a dummy tile: zero fill
        const int tile_x0 = (mt % args.tiles_x) * args.BW;
        const int brow = nt * BN + (int)rank * kBHalf;
        const int kb_lo = z * args.kb_per_split;
        const int kb_hi = min(args.total_kb, kb_lo + args.kb_per_split);
        int g = 0;  // index of the first stage of segment si
        for (int si = 0; si < args.nseg && ok && g < kb_hi; g += kseg_stages(args.seg[si]), ++si) {
          const KSeg sg = args.seg[si];
          const int nst = kseg_stages(sg);
          for (int js = max(0, kb_lo - g); js < nst && g + js < kb_hi; ++js) {
            if (!waited) {
              pdl_wait();
              after_wait();
              waited = true;
            }
            if (q >= (uint32_t)STAGES && !mbar_wait(&empty_bar[s], ph ^ 1, abort_flag, args.err)) {
              ok = false;
              break;
            }
            uint8_t* a_dst = smem + s * stage_bytes;
            uint8_t* b_dst = a_dst + args.a_bytes;
            const int j = js * sg.per;  // first channel block of this stage
            if (sg.taps == 3) {
              if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * tall_bytes);
              tma2_load_4d(a_dst, &maps.at[sg.amap], &full_bar[s], sg.c0 + j * kBK, tile_x0 + sg.dx, tile_y0 - 1,
                           sg.z);
#pragma unroll
              for (int t = 0; t < 3; ++t)
                tma2_load_2d(b_dst + t * kBTileBytes, &maps.b[sg.bmap], &full_bar[s], sg.bk0 + t * sg.bstep + j * kBK,
                             brow);
            } else {
              const int nsub = min(sg.per, sg.nkb - j);
              if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * nsub * single_bytes);
              for (int h = 0; h < nsub; ++h) {
                tma2_load_4d(a_dst + h * kATileBytes, &maps.a[sg.amap], &full_bar[s], sg.c0 + (j + h) * kBK,
                             tile_x0 + sg.dx, tile_y0 + sg.dy, sg.z);
                tma2_load_2d(b_dst + h * kBTileBytes, &maps.b[sg.bmap], &full_bar[s], sg.bk0 + (j + h) * kBK, brow);
              }
            }
            ++q;
            if (++s == STAGES) {
              s = 0;
              ph ^= 1;
            }
          }
        }
      }
    }
    if (lane == 0 && !waited) {
      // no stage issued (no work unit, or the timeout test): wait all the same
      pdl_wait();
      after_wait();
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0 && !*abort_flag) {
      const uint32_t view_bytes = (uint32_t)args.BW * kBK * 2;  // one pixel row of the tall box
      int s = 0;
      uint32_t ph = 0;
      int it = 0;
      bool ok = true;
      for (int u = cluster_id; u < args.units && ok; u += nclusters, ++it) {
        const int z = u % args.splits;
        const int kb_lo = z * args.kb_per_split;
        const int kb_hi = min(args.total_kb, kb_lo + args.kb_per_split);
        const int b = it & 1;
        // the epilogues of both CTAs must have drained this accumulator (first use passes)
        if (!mbar_wait(&acc_empty[b], ((it >> 1) & 1) ^ 1, abort_flag, args.err)) break;
        tc_fence_after();
        const uint32_t tacc = tmem_base + (uint32_t)(b * 256);
        uint32_t acc = 0;  // the first MMA of a unit overwrites the accumulator
        int g = 0;
        for (int si = 0; si < args.nseg && ok && g < kb_hi; g += kseg_stages(args.seg[si]), ++si) {
          const KSeg& sg = args.seg[si];
          const int nst = kseg_stages(sg);
          for (int js = max(0, kb_lo - g); js < nst && g + js < kb_hi; ++js) {
            // operand pairs of this stage: three taps of one box, or up to `per` channel blocks
            const int npair = sg.taps == 3 ? 3 : min(sg.per, sg.nkb - js * sg.per);
            const uint32_t a_step = sg.taps == 3 ? view_bytes : (uint32_t)kATileBytes;
            if (!mbar_wait(&full_bar[s], ph, abort_flag, args.err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * stage_bytes);
            const uint32_t b_addr = a_addr + (uint32_t)args.a_bytes;
            for (int t = 0; t < npair; ++t) {
              const uint64_t adesc = umma_desc_k_sw128(a_addr + (uint32_t)t * a_step);
              const uint64_t bdesc = umma_desc_k_sw128(b_addr + (uint32_t)(t * kBTileBytes));
#pragma unroll
              for (int k = 0; k < kBK / 16; ++k) {
                // +32 bytes along K inside the 128-byte swizzle row = +2 in the encoded address
                umma2_bf16(tacc, adesc + 2 * k, bdesc + 2 * k, kIdesc, acc);
                acc = 1;
              }
            }
            umma2_commit_both(&empty_bar[s]);
            if (++s == STAGES) {
              s = 0;
              ph ^= 1;
            }
          }
        }
        if (ok) umma2_commit_both(&acc_full[b]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    // Every argument the loop needs is copied to registers once: reads of the
    // kernel parameters inside the unrolled loops cannot be hoisted past the
    // global stores by the compiler and would be repeated per element.
    const int N = args.N, Ho = args.Ho, Wo = args.Wo, BH = args.BH, BW = args.BW;
    const int tiles_x = args.tiles_x, tiles_m = args.tiles_m, tiles_n = args.tiles_n, splits = args.splits;
    const int units = args.units;
    float* const partial = args.partial;
    const __nv_bfloat16* const bias = args.epi.bias;
    const __nv_bfloat16* const bias2 = args.epi.bias2;
    const float* const colvec = args.epi.colvec;
    const __nv_bfloat16* const residual = args.epi.residual;
    const int ld_res = args.epi.ld_res, ld_out = args.epi.ld_out, f16_begin = args.epi.f16_begin;
    const bool geglu = args.epi.mode == GEMM_GEGLU;
    const bool f32_out = args.epi.mode == GEMM_F32;
    __nv_bfloat16* const out = args.epi.out;
    const bool has_cols = partial == nullptr && (bias || bias2 || colvec);
    unsigned long long* const rowstat_out = args.epi.rowstat_out;
    const unsigned long long* const rowstat_in = partial ? nullptr : args.epi.rowstat_in;
    const float* const colscale = args.epi.colscale;
    const double ln_inv = args.epi.ln_cols > 0 ? 1.0 / args.epi.ln_cols : 0.0;
    const float ln_eps = args.epi.ln_eps;
    // 32-byte stores and residual loads when every row segment of a chunk starts on a
    // 32-byte boundary (each thread writes a row: one sector per instruction)
    const bool out32 = ((reinterpret_cast<uintptr_t>(out) | ((uintptr_t)ld_out * 2)) & 31) == 0;
    const bool res32 = ((reinterpret_cast<uintptr_t>(residual) | ((uintptr_t)ld_res * 2)) & 31) == 0;
    const bool f32out32 = partial ? (N % 8 == 0 && (reinterpret_cast<uintptr_t>(partial) & 31) == 0)
                                  : (((reinterpret_cast<uintptr_t>(out) | ((uintptr_t)ld_out * 4)) & 31) == 0);

    const int et = threadIdx.x - 64;  // 0..255
    const int half = (warp - 2) >> 2;  // which alternate 32-column chunks this warp handles
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t leader_empty0 = map_to_rank(smem_u32(&acc_empty[0]), 0);
    const uint32_t leader_empty1 = map_to_rank(smem_u32(&acc_empty[1]), 0);
    int it = 0;
    for (int u = cluster_id; u < units; u += nclusters, ++it) {
      const int z = u % splits;
      const int rest = u / splits;
      const int nt = rest % tiles_n;
      const int mt = (rest / tiles_n) * 2 + (int)rank;
      const int n0 = nt * BN;
      const int b = it & 1;
      float* const ecol = epi_col + b * 256;
      float* const escl = epi_scl + b * 256;
      if (rowstat_in) {
        for (int c = et; c < BN; c += kEpiThreads) {
          const int n = n0 + c;
          escl[c] = n < N ? colscale[n] : 0.f;
        }
        if (!has_cols) asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
      }
      if (has_cols) {
        // per-column terms of this unit (biases + FP32 column vector), computed
        // while the main loop runs; buffer b was last read two units ago
        for (int c = et; c < BN; c += kEpiThreads) {
          const int n = n0 + c;
          float a = 0.f;
          if (n < N) {
            if (bias) a += __bfloat162float(bias[n]);
            if (bias2) a += __bfloat162float(bias2[n]);
            if (colvec) a += colvec[n];
          }
          ecol[c] = a;
        }
        asm volatile("bar.sync 2, %0;" ::"n"(kEpiThreads) : "memory");
      }
      const int oy = (mt / tiles_x) * BH + row / BW;
      const int ox = (mt % tiles_x) * BW + row % BW;
      const bool in_image = mt < tiles_m && oy < Ho && ox < Wo;
      const long grow = (long)oy * Wo + ox;
      // LayerNorm of this row from its fixed-point sums (final before this kernel
      // started), computed while the main loop runs: v = rstd*acc - rstd*mean*colscale + colvec
      float ln_a = 1.f, ln_b = 0.f;
      if (rowstat_in && in_image) {
        const double s1 = (double)(long long)__ldcg(rowstat_in + 2 * grow) * (1.0 / kRowSumScale);
        const double s2 = (double)(long long)__ldcg(rowstat_in + 2 * grow + 1) * (1.0 / kRowSqScale);
        const double mean = s1 * ln_inv;
        const double var = fmax(s2 * ln_inv - mean * mean, 0.0);
        const float rstd = (float)(1.0 / sqrt(var + (double)ln_eps));
        ln_a = rstd;
        ln_b = (float)(-mean) * rstd;
      }
      const bool have = mbar_wait(&acc_full[b], (it >> 1) & 1, abort_flag, args.err);
      tc_fence_after();
      const bool valid = have && in_image;
      float rs1 = 0.f, rs2 = 0.f;  // this thread's part of the row sums of the stored output
      const uint32_t tacc = tmem_base + (uint32_t)(b * 256) + lane_off;
      if (half >= kChunks) {
        // no chunk for this warp (BN = 32): still take part in the release
        tc_fence_before();
        asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
      }
      // TMEM reads run one chunk ahead of the arithmetic and stores
      uint32_t rn[32];
      if (half < kChunks) tmem_ld_32x32b_x32(tacc + half * 32, rn);
#pragma unroll 1
      for (int cc = half; cc < kChunks; cc += 2) {
        tmem_ld_wait_regs(rn);
        float v[32];
        {
          const uint32_t ecol_s = smem_u32(ecol + cc * 32), escl_s = smem_u32(escl + cc * 32);
          if (rowstat_in) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 sc = lds_f4(escl_s + 4 * j);
              const float4 co = has_cols ? lds_f4(ecol_s + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
              float t0, t1, t2, t3;  // ln_b * colscale + colvec, then ln_a * acc + that
              fma2v(ln_b, ln_b, sc.x, sc.y, co.x, co.y, t0, t1);
              fma2v(ln_b, ln_b, sc.z, sc.w, co.z, co.w, t2, t3);
              fma2v(ln_a, ln_a, __uint_as_float(rn[j]), __uint_as_float(rn[j + 1]), t0, t1, v[j], v[j + 1]);
              fma2v(ln_a, ln_a, __uint_as_float(rn[j + 2]), __uint_as_float(rn[j + 3]), t2, t3, v[j + 2], v[j + 3]);
            }
          } else if (has_cols) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 co = lds_f4(ecol_s + 4 * j);
              add2(__uint_as_float(rn[j]), __uint_as_float(rn[j + 1]), co.x, co.y, v[j], v[j + 1]);
              add2(__uint_as_float(rn[j + 2]), __uint_as_float(rn[j + 3]), co.z, co.w, v[j + 2], v[j + 3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(rn[j]);
          }
        }
        if (cc + 2 < kChunks) tmem_ld_32x32b_x32(tacc + (cc + 2) * 32, rn);
        if (cc + 2 >= kChunks) {
          // this warp's last read of the accumulator: once all epilogue warps
          // are here it goes back to the MMA issuer
          tc_fence_before();
          asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
          if (warp == 2 && lane == 0) mbar_arrive_cluster(b ? leader_empty1 : leader_empty0);
        }
        if (!valid) continue;
        const int nb = n0 + cc * 32;
        if (nb >= N) continue;
        const bool full = (nb + 32 <= N);
        if (partial || f32_out) {
          float* dst = partial ? partial + ((size_t)z * Ho * Wo + grow) * N + nb
                               : reinterpret_cast<float*>(out) + grow * ld_out + nb;
          if (full && f32out32) {
#pragma unroll
            for (int w = 0; w < 4; ++w)
              st_global_v8(dst + 8 * w, __float_as_uint(v[8 * w]), __float_as_uint(v[8 * w + 1]),
                           __float_as_uint(v[8 * w + 2]), __float_as_uint(v[8 * w + 3]), __float_as_uint(v[8 * w + 4]),
                           __float_as_uint(v[8 * w + 5]), __float_as_uint(v[8 * w + 6]), __float_as_uint(v[8 * w + 7]));
          } else if (full) {
            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
            for (int w = 0; w < 8; ++w) d4[w] = make_float4(v[4 * w], v[4 * w + 1], v[4 * w + 2], v[4 * w + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < N) dst[j] = v[j];
          }
          continue;
        }
        if (geglu) {
          // columns (2j, 2j+1) hold (value_j, gate_j); output column (nb/2 + j)
          uint32_t o[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float a0 = v[4 * j] * gelu_erf(v[4 * j + 1]);
            const float a1 = v[4 * j + 2] * gelu_erf(v[4 * j + 3]);
            o[j] = pack_bf16x2(a0, a1);
          }
          __nv_bfloat16* dst = out + grow * ld_out + (nb >> 1);
          if (full && out32) {
            st_global_v8(dst, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
          } else if (full) {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
            d4[0] = make_uint4(o[0], o[1], o[2], o[3]);
            d4[1] = make_uint4(o[4], o[5], o[6], o[7]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              if (nb + 2 * j < N) {
                const uint32_t w = o[j >> 1];
                dst[j] = __ushort_as_bfloat16((unsigned short)((j & 1) ? (w >> 16) : (w & 0xFFFF)));
              }
            }
          }
          continue;
        }
        if (residual) {
          const __nv_bfloat16* rs = residual + grow * ld_res + nb;
          if (full && res32) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              uint32_t w[8];
              ld_global_v8(rs + 16 * h, w);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                add2(v[16 * h + 2 * i], v[16 * h + 2 * i + 1], bf16lo(w[i]), bf16hi(w[i]), v[16 * h + 2 * i],
                     v[16 * h + 2 * i + 1]);
            }
          } else if (full) {
            const uint4* r4 = reinterpret_cast<const uint4*>(rs);
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              const uint4 w = r4[w4];
              v[8 * w4 + 0] += bf16lo(w.x);
              v[8 * w4 + 1] += bf16hi(w.x);
              v[8 * w4 + 2] += bf16lo(w.y);
              v[8 * w4 + 3] += bf16hi(w.y);
              v[8 * w4 + 4] += bf16lo(w.z);
              v[8 * w4 + 5] += bf16hi(w.z);
              v[8 * w4 + 6] += bf16lo(w.w);
              v[8 * w4 + 7] += bf16hi(w.w);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (nb + j < N) v[j] += __bfloat162float(rs[j]);
          }
        }
        __nv_bfloat16* dst = out + grow * ld_out + nb;
        if (full && f16_begin > 0 && nb >= f16_begin) {
          // FP16 columns (the attention values V; no row statistics are taken over them)
          uint32_t o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = pack_f16x2(v[2 * i], v[2 * i + 1]);
          if (out32) {
            st_global_v8(dst, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
            st_global_v8(dst + 16, o[8], o[9], o[10], o[11], o[12], o[13], o[14], o[15]);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int w = 0; w < 4; ++w) d4[w] = make_uint4(o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
          }
        } else if (full) {
          uint32_t o[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          if (out32) {
            st_global_v8(dst, o[0], o[1], o[2], o[3], o[4], o[5], o[6], o[7]);
            st_global_v8(dst + 16, o[8], o[9], o[10], o[11], o[12], o[13], o[14], o[15]);
          } else {
            uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
            for (int w = 0; w < 4; ++w) d4[w] = make_uint4(o[4 * w], o[4 * w + 1], o[4 * w + 2], o[4 * w + 3]);
          }
          if (rowstat_out) {
            // sums of the stored BF16 values, read back from the packed words
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float lo = bf16lo(o[i]), hi = bf16hi(o[i]);
              rs1 += lo + hi;
              rs2 = fmaf(lo, lo, fmaf(hi, hi, rs2));
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            if (nb + j < N) {
              const __nv_bfloat16 q = __float2bfloat16_rn(v[j]);
              dst[j] = q;
              if (rowstat_out) {
                rs1 += __bfloat162float(q);
                rs2 = fmaf(__bfloat162float(q), __bfloat162float(q), rs2);
              }
            }
          }
        }
      }
      if (rowstat_out && !partial && valid && half < kChunks) {
        // integer adds: the sums do not depend on the order in which units arrive
        atomicAdd(rowstat_out + 2 * grow, (unsigned long long)llrint((double)rs1 * kRowSumScale));
        atomicAdd(rowstat_out + 2 * grow + 1, (unsigned long long)llrint((double)rs2 * kRowSqScale));
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) tmem_dealloc_2sm(tmem_base, kTmemCols);
}

// Split-K reduction of 8 columns (row, c .. c+7): sum over splits of the FP32
// partials in split order (deterministic), then the epilogue. Returns, through
// rs1 / rs2, the sums of the stored BF16 values (plain stores only).
__device__ __forceinline__ void splitk_reduce_vec(const float* __restrict__ partial, int splits, int M, int N,
                                                  const GemmEpi& epi, int row, int c, float& rs1, float& rs2) {
  // the splits' partials are requested four at a time before any is added; the
  // sum still runs in split order, so the result does not depend on the grouping
  float v[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const size_t zstride = (size_t)M * N;
  const float* base = partial + (size_t)row * N + c;
  for (int z0 = 0; z0 < splits; z0 += 4) {
    float4 a[4], b[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (z0 + u < splits) {
        const float4* pz = reinterpret_cast<const float4*>(base + (size_t)(z0 + u) * zstride);
        a[u] = __ldcg(pz);
        b[u] = __ldcg(pz + 1);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (z0 + u < splits) {
        if (z0 + u == 0) {
          v[0] = a[u].x; v[1] = a[u].y; v[2] = a[u].z; v[3] = a[u].w;
          v[4] = b[u].x; v[5] = b[u].y; v[6] = b[u].z; v[7] = b[u].w;
        } else {
          v[0] += a[u].x; v[1] += a[u].y; v[2] += a[u].z; v[3] += a[u].w;
          v[4] += b[u].x; v[5] += b[u].y; v[6] += b[u].z; v[7] += b[u].w;
        }
      }
    }
  }
  if (epi.rowstat_in) {
    // folded LayerNorm: rstd * acc - rstd * mean * colscale + colvec
    const double s1 = (double)(long long)__ldcg(epi.rowstat_in + 2 * row) * (1.0 / kRowSumScale);
    const double s2 = (double)(long long)__ldcg(epi.rowstat_in + 2 * row + 1) * (1.0 / kRowSqScale);
    const double inv = 1.0 / epi.ln_cols;
    const double mean = s1 * inv;
    const double var = fmax(s2 * inv - mean * mean, 0.0);
    const float rstd = (float)(1.0 / sqrt(var + (double)epi.ln_eps));
    const float lb = (float)(-mean) * rstd;
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = fmaf(rstd, v[j], lb * epi.colscale[c + j]);
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
    return;
  }
  if (epi.residual) {
    const uint4 r = *reinterpret_cast<const uint4*>(epi.residual + (size_t)row * epi.ld_res + c);
    v[0] += bf16lo(r.x); v[1] += bf16hi(r.x); v[2] += bf16lo(r.y); v[3] += bf16hi(r.y);
    v[4] += bf16lo(r.z); v[5] += bf16hi(r.z); v[6] += bf16lo(r.w); v[7] += bf16hi(r.w);
  }
  if (epi.f16_begin > 0 && c >= epi.f16_begin) {
    *reinterpret_cast<uint4*>(epi.out + (size_t)row * epi.ld_out + c) =
        make_uint4(pack_f16x2(v[0], v[1]), pack_f16x2(v[2], v[3]), pack_f16x2(v[4], v[5]), pack_f16x2(v[6], v[7]));
    return;
  }
  const uint4 o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                             pack_bf16x2(v[6], v[7]));
  *reinterpret_cast<uint4*>(epi.out + (size_t)row * epi.ld_out + c) = o;
  const uint32_t w[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = bf16lo(w[j]), hi = bf16hi(w[j]);
    rs1 += lo + hi;
    rs2 = fmaf(lo, lo, fmaf(hi, hi, rs2));
  }
}

// Split-K reduction: out = epilogue(sum over splits of partial), 8 columns per
// thread. With row statistics requested, each warp takes one 256-column segment
// of one row and adds its shuffle-reduced sums into the row's fixed-point pair.
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N, GemmEpi epi) {
  pdl_wait();
  pdl_trigger();
  const int V = N / 8;
  if (!epi.rowstat_out) {
    const size_t total = (size_t)M * V;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
      float r1 = 0.f, r2 = 0.f;
      splitk_reduce_vec(partial, splits, M, N, epi, (int)(i / V), (int)(i % V) * 8, r1, r2);
    }
    return;
  }
  const int lane = threadIdx.x & 31;
  const int segs = (V + 31) / 32;
  const size_t warps = (size_t)M * segs;
  const size_t nwarps = (size_t)gridDim.x * (blockDim.x >> 5);
  for (size_t wi = blockIdx.x * (size_t)(blockDim.x >> 5) + (threadIdx.x >> 5); wi < warps; wi += nwarps) {
    const int row = (int)(wi / segs);
    const int vec = (int)(wi % segs) * 32 + lane;
    float r1 = 0.f, r2 = 0.f;
    if (vec < V) splitk_reduce_vec(partial, splits, M, N, epi, row, vec * 8, r1, r2);
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      r1 += __shfl_xor_sync(0xffffffffu, r1, o);
      r2 += __shfl_xor_sync(0xffffffffu, r2, o);
    }
    if (lane == 0) {
      atomicAdd(epi.rowstat_out + 2 * row, (unsigned long long)llrint((double)r1 * kRowSumScale));
      atomicAdd(epi.rowstat_out + 2 * row + 1, (unsigned long long)llrint((double)r2 * kRowSqScale));
    }
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

template <int BN>
static int launch_bn(const GemmMaps& maps, const GemmArgs& args, int grid, size_t smem, cudaStream_t st) {
  static bool attr_set = false;  // benign race: the attribute value is identical for every caller
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    if (e != cudaSuccess) return (int)e;
    attr_set = true;
  }
  return (int)launch_pdl(gemm_tc_kernel<BN>, dim3(grid), dim3(kGemmThreads), smem, st, maps, args);
}

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

// CTA pairs that can be resident at once (a GPC with an odd number of SMs
// leaves one SM out of every pairing).
static int max_active_clusters() {
  static int n = 0;
  if (n == 0) {
    cudaFuncSetAttribute(gemm_tc_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count() / 2));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = 200 * 1024;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, gemm_tc_kernel<256>, &cfg) != cudaSuccess || c <= 0) {
      cudaGetLastError();
      c = sm_count() / 2;
    }
    n = std::min(c, sm_count() / 2);
  }
  return n;
}

// Output tile rectangle of 128 pixels (BW x BH) with the fewest tiles. With
// foldable 3x3 taps, narrow-and-tall rectangles come first: the shared box of
// a tap column holds (BH + 2) rows for 3*BH rows of work.
static void choose_tile_rect(int Ho, int Wo, bool prefer_tall, int* BH, int* BW) {
  if (Ho == 1) {
    *BH = 1;
    *BW = 128;
    return;
  }
  int best = -1, bw_best = 16;
  const int plain[] = {16, 32, 8, 64, 4, 128};
  const int tall[] = {8, 16, 32, 64, 4, 128};
  for (int bw : prefer_tall ? tall : plain) {
    const int bh = 128 / bw;
    const int tiles = ((Wo + bw - 1) / bw) * ((Ho + bh - 1) / bh);
    if (best < 0 || tiles < best) {
      best = tiles;
      bw_best = bw;
    }
  }
  *BW = bw_best;
  *BH = 128 / bw_best;
}

// Kernel segments of a problem: every group of three taps that differ only in
// dy = -1, 0, +1 (same source, column, plane, channels and length, B offsets
// bk0, bk0 + S, bk0 + 2S) becomes one 3-tap segment when `fold` is set.
static int build_ksegs(const GemmProblem& p, bool fold, KSeg* out) {
  bool used[kGemmMaxSeg] = {};
  int n = 0;
  for (int i = 0; i < p.nseg; ++i) {
    if (used[i]) continue;
    const GemmSeg& a = p.seg[i];
    int mid = -1, hi = -1;
    if (fold && a.dy == -1) {
      for (int j = 0; j < p.nseg; ++j) {
        const GemmSeg& c = p.seg[j];
        if (used[j] || j == i || c.amap != a.amap || c.bmap != a.bmap || c.dx != a.dx || c.z != a.z ||
            c.c0 != a.c0 || c.nkb != a.nkb)
          continue;
        if (c.dy == 0 && mid < 0) mid = j;
      }
      if (mid >= 0) {
        const int S = p.seg[mid].bk0 - a.bk0;
        for (int j = 0; j < p.nseg; ++j) {
          const GemmSeg& c = p.seg[j];
          if (used[j] || j == i || j == mid || c.amap != a.amap || c.bmap != a.bmap || c.dx != a.dx ||
              c.z != a.z || c.c0 != a.c0 || c.nkb != a.nkb || c.dy != 1 || c.bk0 != a.bk0 + 2 * S)
            continue;
          hi = j;
          break;
        }
      }
    }
    KSeg& k = out[n++];
    k.amap = a.amap;
    k.bmap = a.bmap;
    k.dx = a.dx;
    k.dy = a.dy;
    k.z = a.z;
    k.c0 = a.c0;
    k.bk0 = a.bk0;
    k.nkb = a.nkb;
    k.taps = 1;
    k.bstep = 0;
    k.per = a.nkb >= 2 ? 2 : 1;
    if (mid >= 0 && hi >= 0) {
      k.taps = 3;
      k.bstep = p.seg[mid].bk0 - a.bk0;
      k.per = 1;
      used[mid] = used[hi] = true;
    }
    used[i] = true;
  }
  return n;
}

struct GemmPlan {
  int BH, BW, tiles_x, tiles_m, bn, tiles_n, splits, kb_per_split, total_kb, units, clusters;
  int nkseg, stages, stage_bytes, a_bytes;
  bool tall;
  KSeg kseg[kGemmMaxSeg];
};

// Shared-memory layout of a stage for N tile bn: the A region holds the
// largest A operand of any segment (a tall box, or `per` boxes), the B region
// the largest number of B slices.
static void stage_layout(const GemmPlan& g, int bn, int* a_bytes, int* stage_bytes, int* stages) {
  const int tall_a = ((g.BH + 2) * g.BW * kBK * 2 + 1023) & ~1023;
  int a = kATileBytes, nb = 1;
  for (int i = 0; i < g.nkseg; ++i) {
    const KSeg& k = g.kseg[i];
    if (k.taps == 3) {
      a = std::max(a, tall_a);
      nb = std::max(nb, 3);
    } else {
      a = std::max(a, k.per * kATileBytes);
      nb = std::max(nb, k.per);
    }
  }
  *a_bytes = a;
  *stage_bytes = a + nb * (bn / 2) * kBK * 2;
  *stages = std::min(kMaxStages, (kSmemLimit - kSmemFixed) / *stage_bytes);
}

// Estimated cycles of a plan. A CTA pair performs 2*256*BN*64 FLOPs per tap
// and k-block (2*BN cycles per SM at the tensor rate); each SM takes its A box
// and BN/2 rows of B per stage at about 50 bytes per cycle from L2, so a stage
// costs the slower of the two. Units are spread over the clusters in rounds;
// the split-K reduction is added on top.
static double plan_cost(const GemmPlan& g, int bn, int splits, int pairs, int N, long M, int clusters) {
  const int tiles_n = (N + bn - 1) / bn;
  const long units = (long)pairs * tiles_n * splits;
  const long rounds = (units + clusters - 1) / clusters;
  double unit_cycles = 0;
  const int a_tall = (g.BH + 2) * g.BW * kBK * 2;
  for (int i = 0; i < g.nkseg; ++i) {
    const KSeg& k = g.kseg[i];
    // operand pairs per stage and the MMA cycles of one (a K=16 MMA takes at least ~54 cycles)
    const int pairs_per_stage = k.taps == 3 ? 3 : k.per;
    const double mma = pairs_per_stage * 4.0 * std::max(54.0, bn / 2.0);
    const double load =
        ((k.taps == 3 ? a_tall : k.per * kATileBytes) + pairs_per_stage * (bn / 2) * kBK * 2.0) / 50.0;
    unit_cycles += kseg_stages(k) * std::max(std::max(mma, load), 520.0);  // 520: stage handshake
  }
  unit_cycles /= splits;
  const double epilogue = 40.0 * bn;  // 8 warps drain 128 x BN FP32 values and store them
  double cost = (double)rounds * (unit_cycles + 600.0) + epilogue;
  if (rounds > 1) cost += (double)(rounds - 1) * std::max(0.0, epilogue - unit_cycles);
  if (splits > 1) cost += 4000.0 + (double)splits * M * N * 4.0 / 3000.0;
  return cost;
}

// Tile shape, N tile and split-K factor for a problem.
static bool plan_gemm(const GemmProblem& p, GemmPlan* g) {
  KSeg probe[kGemmMaxSeg];
  bool foldable = false;
  {
    const int n = build_ksegs(p, true, probe);
    for (int i = 0; i < n; ++i) foldable |= probe[i].taps == 3;
  }
  choose_tile_rect(p.Ho, p.Wo, foldable, &g->BH, &g->BW);
  g->tall = foldable && g->BH >= 2 && g->BW % 8 == 0 && g->BW <= 16;
  g->nkseg = build_ksegs(p, g->tall, g->kseg);
  bool any_tall = false;
  for (int i = 0; i < g->nkseg; ++i) any_tall |= g->kseg[i].taps == 3;
  if (any_tall) {
    // the few single blocks beside tall stages (a fused 1x1 shortcut) keep one
    // block per stage so the stage stays at the tall size
    for (int i = 0; i < g->nkseg; ++i)
      if (g->kseg[i].taps == 1) g->kseg[i].per = 1;
  }
  g->tiles_x = (p.Wo + g->BW - 1) / g->BW;
  g->tiles_m = g->tiles_x * ((p.Ho + g->BH - 1) / g->BH);
  g->total_kb = 0;
  for (int i = 0; i < g->nkseg; ++i) g->total_kb += kseg_stages(g->kseg[i]);
  if (g->total_kb <= 0) return false;
  const int pairs = (g->tiles_m + 1) / 2;
  const int max_clusters = max_active_clusters();
  const long M = (long)p.Ho * p.Wo;
  const size_t per_split = (size_t)M * p.N * sizeof(float);
  const int bns[] = {256, 224, 192, 160, 128, 96, 64, 32};
  const int sps[] = {1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15, 16};
  double best = -1.0;
  g->bn = 0;
  g->splits = 1;
  for (int bn : bns) {
    if (p.force_bn) {
      if (bn != p.force_bn) continue;
    } else {
      if (bn > 32 && p.N <= bn / 2) continue;  // more than half the tile would be padding
      if (bn == 32 && p.N > 64) continue;
    }
    for (int sp : sps) {
      if (p.force_splits) {
        if (sp != std::min(p.force_splits, g->total_kb)) continue;
      } else if (sp > 1 && (g->total_kb / sp < 2 || (sp > 8 && sp % 2))) {
        continue;
      }
      if (sp > 1 && (!p.splitk_ws || per_split * sp > p.splitk_ws_bytes || p.N % 8 || p.epi.mode == GEMM_F32))
        continue;
      const double c = plan_cost(*g, bn, sp, pairs, p.N, M, max_clusters);
      if (best < 0 || c < best) {
        best = c;
        g->bn = bn;
        g->splits = sp;
      }
    }
  }
  if (g->bn == 0) return false;
  g->tiles_n = (p.N + g->bn - 1) / g->bn;
  g->kb_per_split = (g->total_kb + g->splits - 1) / g->splits;
  g->splits = (g->total_kb + g->kb_per_split - 1) / g->kb_per_split;  // no empty split
  g->units = pairs * g->tiles_n * g->splits;
  g->clusters = std::min(g->units, max_clusters);
  stage_layout(*g, g->bn, &g->a_bytes, &g->stage_bytes, &g->stages);
  return g->stages >= 2;
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
  args.tiles_m = g.tiles_m;
  args.N = p.N;
  args.nseg = g.nkseg;
  for (int i = 0; i < g.nkseg; ++i) args.seg[i] = g.kseg[i];
  args.total_kb = g.total_kb;
  args.kb_per_split = g.kb_per_split;
  args.splits = g.splits;
  args.tiles_n = g.tiles_n;
  args.units = g.units;
  args.stages = g.stages;
  args.stage_bytes = g.stage_bytes;
  args.a_bytes = g.a_bytes;
  args.epi = p.epi;
  args.partial = g.splits > 1 ? p.splitk_ws : nullptr;
  args.err = p.err;
  args.hold_spins = p.hold_spins;
  const int bn = g.bn;

  GemmMaps maps;
  memset(&maps, 0, sizeof(maps));
  for (int i = 0; i < kGemmMaxA; ++i) {
    const GemmASrc& a = p.a[i < p.na ? i : 0];
    uint64_t d[4] = {(uint64_t)a.C, (uint64_t)a.W, (uint64_t)a.H, (uint64_t)a.Z};
    if (!tmap_encode_4d(&maps.a[i], a.ptr, d, args.BW, args.BH)) return -2;
    if (g.tall) {
      if (!tmap_encode_4d(&maps.at[i], a.ptr, d, args.BW, args.BH + 2)) return -2;
    } else {
      maps.at[i] = maps.a[i];
    }
  }
  for (int i = 0; i < kGemmMaxB; ++i) {
    const GemmBSrc& b = p.b[i < p.nb ? i : 0];
    if (!tmap_encode_2d(&maps.b[i], b.ptr, (uint64_t)b.K, (uint64_t)b.rows, 64, (uint32_t)(bn / 2))) return -2;
  }
  const int grid = 2 * g.clusters;
  const size_t smem = (size_t)kSmemFixed + (size_t)g.stages * g.stage_bytes;
  int e;
  switch (bn) {
    case 32: e = launch_bn<32>(maps, args, grid, smem, stream); break;
    case 64: e = launch_bn<64>(maps, args, grid, smem, stream); break;
    case 96: e = launch_bn<96>(maps, args, grid, smem, stream); break;
    case 128: e = launch_bn<128>(maps, args, grid, smem, stream); break;
    case 160: e = launch_bn<160>(maps, args, grid, smem, stream); break;
    case 192: e = launch_bn<192>(maps, args, grid, smem, stream); break;
    case 224: e = launch_bn<224>(maps, args, grid, smem, stream); break;
    case 256: e = launch_bn<256>(maps, args, grid, smem, stream); break;
    default: return -1;
  }
  if (e != 0 || g.splits <= 1) return e;
  const int M = p.Ho * p.Wo;
  const size_t vecs = (size_t)M * (p.N / 8);
  int blocks = (int)((vecs + 255) / 256);
  if (blocks > sm_count() * 8) blocks = sm_count() * 8;
  return (int)launch_pdl(splitk_reduce_kernel, dim3(blocks), dim3(256), 0, stream, (const float*)p.splitk_ws,
                         g.splits, M, p.N, p.epi);
}

}  // namespace sdk
