// Flash attention on the 5th-generation tensor cores (sm_100a), head_dim 64.
//
// What it computes (SD1.5 anatomy page, section 3.4; Transformer2DModel panel,
// section 4 of the SD2.1 page): per head h, O_h = softmax(Q_h K_h^T / 8) V_h for
// self-attention over the H*W image tokens (Q = K = V source) and for
// cross-attention over the 77 context rows.
//
// Work: every (head, 128-query tile) item runs over ceil(Nk/128) key tiles.
// The grid is persistent (two CTAs per SM) and the sequence of all
// (item, key tile) steps is cut into equal contiguous ranges, one per CTA, so
// no SM idles while another finishes a second wave. An item whose key tiles
// are split between CTAs leaves one piece per CTA in a workspace slot (its
// unnormalised output with its running maximum and row sum); a small merge
// kernel then combines the pieces of each split item in CTA order. Splitting is
// used only where it shortens the longest CTA.
//
// 192 threads per CTA:
//   warps 0-3  softmax: thread i owns query row i (TMEM lane i). Per 128-key
//              tile it reads its S row from TMEM, keeps a running maximum in the
//              log2 domain, and forms P = exp2(s*log2e/8 - m) two at a time: the
//              pair of FP32 exponents is rounded to FP16 and one packed
//              ex2.approx.f16x2 gives both probabilities, already in the FP16
//              form the PV product takes. P goes to shared memory (the
//              A operand of the PV product, 128-byte swizzled); the row sum is
//              kept in four packed FP16 partial sums per tile, added into FP32
//              once per tile. The output O lives in TMEM and is rescaled only
//              when the running maximum grew by more than 2^8 since the last
//              rescale (P values stay <= 256). The TMEM accesses are
//              warp-collective, so a warp rescales together when any of its
//              rows needs it (the others with factor 1).
//   warp 4     TMA producer: Q once per item, K tiles (double-buffered) and V
//              tiles (single buffer, reloaded once the previous PV product is
//              done), zero-filled past the last key. V arrives as FP16 (the
//              projection GEMM stores those columns in FP16).
//   warp 5     MMA issuer (one thread): S = Q K^T (M=128, N=128, K=64, BF16) and
//              O += P V (M=128, N=64, K=128, FP16, V read MN-major), both
//              tcgen05.mma kind::f16 with FP32 accumulation in TMEM.
// TMEM: S in columns [0, 128), O in [128, 192) of a 256-column allocation, so
// two CTAs fit on one SM and overlap each other's softmax and MMA phases.
#include "common.cuh"
#include "kernels.cuh"

#include <algorithm>
#include <mutex>

#include "gemm_tc.cuh"

namespace sdk {

namespace {

constexpr int kAQ = 128;        // queries per CTA
constexpr int kAK = 128;        // keys per tile
constexpr int kTileBytes = 128 * 64 * 2;  // one [128 x 64] BF16 tile = 16 KB
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kOCol = 128;

// Instruction descriptor, FP32 accumulator, M = 128, A K-major: BF16 x BF16 with
// B K-major (S = Q K^T), or FP16 x FP16 with B MN-major (O += P V).
__host__ __device__ constexpr uint32_t idesc_attn(int N, bool pv) {
  return (1u << 4) | (pv ? 0u : (1u << 7) | (1u << 10)) | ((pv ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// Shared-memory descriptor of an MN-major operand tile stored as rows of 128
// bytes along K with the 128-byte swizzle: 8-row groups along K are 1024 bytes
// apart (stride byte offset); the MN extent is one 64-element swizzle atom.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;                       // leading byte offset (one MN atom: unused)
  d |= (uint64_t)((1024 >> 4) & 0x3FFF) << 32;  // stride byte offset: next 8 rows along K
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Two FP32 values rounded to one packed FP16 pair (lo in the low half).
__device__ __forceinline__ uint32_t cvt_f16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// 2^x for both halves of a packed FP16 pair (one exponential-unit instruction).
__device__ __forceinline__ uint32_t ex2_f16x2(uint32_t x) {
  uint32_t y;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ uint32_t add_f16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ float f16x2_sum(uint32_t h) {
  const __half2 v = *reinterpret_cast<const __half2*>(&h);
  return __low2float(v) + __high2float(v);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float max3(float a, float b, float c) {
  float y;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
  return y;
}

// (x0, x1) = (s0 * k + c, s1 * k + c) as one packed FP32 FMA (sm_100), each element
// rounded exactly as a scalar fmaf
__device__ __forceinline__ void fma2(float s0, float s1, float k, float c, float& x0, float& x1) {
  asm("{\n\t.reg .b64 t, u, v;\n\t"
      "mov.b64 t, {%2, %3};\n\t"
      "mov.b64 u, {%4, %4};\n\t"
      "mov.b64 v, {%5, %5};\n\t"
      "fma.rn.f32x2 t, t, u, v;\n\t"
      "mov.b64 {%0, %1}, t;\n\t}"
      : "=f"(x0), "=f"(x1)
      : "f"(s0), "f"(s1), "f"(k), "f"(c));
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bounded wait for a softmax warp. tcgen05.ld / tcgen05.st are warp-collective
// (.sync.aligned): every lane of the warp must execute them together. The lanes
// of one warp may leave the polling loop at different polls, and one lane may
// give up while another sees the phase complete; the vote brings them back
// together and gives all of them one answer, so the warp stays or leaves as a
// whole.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
  const bool ok = mbar_wait(bar, parity, abort, err);
  return __all_sync(0xffffffffu, ok);
}

struct __align__(64) AttnMaps {
  CUtensorMap q;
  CUtensorMap kv;
};

struct AttnArgs {
  int32_t Nq, Nk;
  int32_t q_col, k_col, v_col;  // column offsets of head 0 in the Q and KV maps
  __nv_bfloat16* O;
  int32_t ldo;
  float scale_log2;
  int32_t qtiles, ktiles;  // 128-query tiles per head, 128-key tiles per item
  int64_t steps;           // heads * qtiles * ktiles
  int32_t ctas;            // grid size: CTA c runs steps [c*steps/ctas, (c+1)*steps/ctas)
  float* partial;          // [ctas][2] slots of kSlotFloats (pieces of split items)
  int* err;
};

constexpr int kSlotFloats = 128 * 64 + 2 * 128;  // O rows, then running maxima, then row sums

__host__ __device__ inline int64_t cta_first_step(int64_t c, int64_t steps, int64_t ctas) {
  return c * steps / ctas;
}

}  // namespace

// End of a CTA's part of item X (one query row per thread, O in TMEM at
// tOrow): a whole item is normalised and stored as BF16; a piece of a split
// item goes to this CTA's workspace slot (0 for its first item, 1 otherwise)
// for the merge kernel. Kept out of line: it runs once per item and its
// registers would otherwise compete with the S row of the softmax loop.
__device__ __noinline__ void attn_item_end(const AttnArgs& args, uint32_t tOrow, int row, int X, bool whole,
                                           bool first_item, float m_used, float l) {
  const int h = X / args.qtiles;
  const int qrow = (X % args.qtiles) * kAQ + row;
  if (whole) {
    __nv_bfloat16* dst = args.O + (size_t)qrow * args.ldo + h * 64;
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tOrow + c * 32, r);
      tmem_ld_wait();
      if (qrow < args.Nq) {
        uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          d4[u] = make_uint4(pack_bf16x2(__uint_as_float(r[8 * u]) * inv, __uint_as_float(r[8 * u + 1]) * inv),
                             pack_bf16x2(__uint_as_float(r[8 * u + 2]) * inv, __uint_as_float(r[8 * u + 3]) * inv),
                             pack_bf16x2(__uint_as_float(r[8 * u + 4]) * inv, __uint_as_float(r[8 * u + 5]) * inv),
                             pack_bf16x2(__uint_as_float(r[8 * u + 6]) * inv, __uint_as_float(r[8 * u + 7]) * inv));
        }
      }
    }
    return;
  }
  float* slot = args.partial + ((size_t)blockIdx.x * 2 + (first_item ? 0 : 1)) * kSlotFloats;
#pragma unroll 1
  for (int c = 0; c < 2; ++c) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(tOrow + c * 32, r);
    tmem_ld_wait();
    float4* o4 = reinterpret_cast<float4*>(slot + row * 64 + c * 32);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      __stcg(o4 + u, make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                                 __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3])));
  }
  __stcg(slot + 8192 + row, m_used);
  __stcg(slot + 8320 + row, l);
}

__global__ void __launch_bounds__(192, 2)
    attention_tc_kernel(const __grid_constant__ AttnMaps maps, const __grid_constant__ AttnArgs args) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // 16 KB
  uint8_t* sK = sQ + kTileBytes;            // 2 x 16 KB
  uint8_t* sV = sK + 2 * kTileBytes;        // 16 KB
  uint8_t* sP = sV + kTileBytes;            // 2 halves x 16 KB: keys [0,64) and [64,128)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + 2 * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;   // [2]
  uint64_t* k_empty = bars + 3;  // [2]
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 6;
  uint64_t* s_full = bars + 7;
  uint64_t* p_full = bars + 8;
  uint64_t* pv_done = bars + 9;
  uint64_t* s_free = bars + 10;
  uint64_t* q_empty = bars + 11;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = args.ktiles;
  const int w0 = (int)cta_first_step(blockIdx.x, args.steps, args.ctas);  // first step of this CTA
  const int T = (int)cta_first_step(blockIdx.x + 1, args.steps, args.ctas) - w0;  // steps of this CTA

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(&k_full[0], 1);
    mbar_init(&k_full[1], 1);
    mbar_init(&k_empty[0], 1);
    mbar_init(&k_empty[1], 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(s_free, 128);
    mbar_init(q_empty, 1);
    *abort_flag = 0;
    fence_barrier_init();
    // descriptors and arguments are kernel parameters: fetch them into the caches
    // before waiting for the previous kernel
    tma_prefetch_desc(&maps.q);
    tma_prefetch_desc(&maps.kv);
    const int64_t touch = args.steps + args.ctas + args.qtiles + args.ktiles + args.Nq + args.Nk + args.q_col +
                          args.k_col + args.v_col;
    asm volatile("" ::"l"(touch));
  }
  if (warp == 5) tmem_alloc(tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();
  pdl_trigger();
  const uint32_t tS = tmem;
  const uint32_t tO = tmem + kOCol;

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int ii = 0;  // items started
      int X = (int)(w0 / nt), j = (int)(w0 % nt);
      for (int t = 0; t < T; ++t, j = (j + 1 == nt) ? 0 : j + 1, X += (j == 0)) {
        const int h = X / args.qtiles, qt = X % args.qtiles;
        if (t == 0 || j == 0) {
          // Q of a new item once every S product of the previous one is done
          if (ii > 0 && !mbar_wait(q_empty, (ii - 1) & 1, abort_flag, args.err)) break;
          mbar_arrive_expect_tx(q_full, kTileBytes);
          tma_load_2d(sQ, &maps.q, q_full, args.q_col + h * 64, qt * kAQ);
          ++ii;
        }
        const int s = t & 1;
        if (t >= 2 && !mbar_wait(&k_empty[s], ((t >> 1) - 1) & 1, abort_flag, args.err)) break;
        mbar_arrive_expect_tx(&k_full[s], kTileBytes);
        tma_load_2d(sK + s * kTileBytes, &maps.kv, &k_full[s], args.k_col + h * 64, j * kAK);
        if (t >= 1 && !mbar_wait(v_empty, (t - 1) & 1, abort_flag, args.err)) break;
        mbar_arrive_expect_tx(v_full, kTileBytes);
        tma_load_2d(sV, &maps.kv, v_full, args.v_col + h * 64, j * kAK);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_attn(128, false);
      constexpr uint32_t kIdO = idesc_attn(64, true);
      const uint64_t qdesc = umma_desc_k_sw128(smem_u32(sQ));
      int ii = 0;                // items whose Q has been waited for
      int jS = (int)(w0 % nt);   // key tile of S_t
      int jP = jS;               // key tile of the PV product of step t - 1
      // step t issues S_t (once the softmax warps hold S_{t-1} in registers), then
      // O += P_{t-1} V_{t-1}
      for (int t = 0; t <= T; ++t) {
        if (t < T) {
          if (t > 0 && !mbar_wait(s_free, (t - 1) & 1, abort_flag, args.err)) break;
          if (t == 0 || jS == 0) {
            if (!mbar_wait(q_full, ii & 1, abort_flag, args.err)) break;
            ++ii;
          }
          const int s = t & 1;
          if (!mbar_wait(&k_full[s], (t >> 1) & 1, abort_flag, args.err)) break;
          tc_fence_after();
          const uint64_t kdesc = umma_desc_k_sw128(smem_u32(sK + s * kTileBytes));
#pragma unroll
          for (int k = 0; k < 4; ++k) umma_bf16(tS, qdesc + 2 * k, kdesc + 2 * k, kIdS, k > 0 ? 1u : 0u);
          umma_commit(&k_empty[s]);
          umma_commit(s_full);
          if (t == T - 1 || jS == nt - 1) umma_commit(q_empty);  // last S of this item
          jS = (jS + 1 == nt) ? 0 : jS + 1;
        }
        if (t > 0) {
          const int tp = t - 1;
          if (!mbar_wait(p_full, tp & 1, abort_flag, args.err)) break;
          if (!mbar_wait(v_full, tp & 1, abort_flag, args.err)) break;
          tc_fence_after();
          const bool first = tp == 0 || jP == 0;
          const uint32_t vbase = smem_u32(sV);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // keys [16k, 16k + 16): P half k/4 at +32 bytes per step; V rows 16k.. (+2048 bytes per step)
            const uint64_t pdesc = umma_desc_k_sw128(smem_u32(sP + (k >> 2) * kTileBytes)) + 2 * (k & 3);
            const uint64_t vdesc = umma_desc_mn_sw128(vbase + k * 2048);
            umma_bf16(tO, pdesc, vdesc, kIdO, (!first || k > 0) ? 1u : 0u);
          }
          umma_commit(v_empty);
          umma_commit(pv_done);
          jP = (jP + 1 == nt) ? 0 : jP + 1;
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax warps 0-3
    const int row = threadIdx.x;  // TMEM lane == query row within the tile
    const uint32_t tSrow = tS + ((uint32_t)(warp * 32) << 16);  // this warp's lane quarter
    const uint32_t tOrow = tO + ((uint32_t)(warp * 32) << 16);
    const float sl2 = args.scale_log2;
    float m_used = -INFINITY;  // maximum the stored P and O are relative to (log2 domain)
    float l = 0.f;
    const uint32_t prow0 = smem_u32(sP) + row * 128;  // this row of P, 32-bit shared address
    int j = (int)(w0 % nt);  // key tile of step t within its item
    for (int t = 0; t < T; ++t, j = (j + 1 == nt) ? 0 : j + 1) {
      const bool first = t == 0 || j == 0;
      const bool last = t == T - 1 || j == nt - 1;
      if (!mbar_wait_warp(s_full, t & 1, abort_flag, args.err)) break;
      tc_fence_after();
      const int kvalid = args.Nk - j * kAK;  // keys of this tile that exist
      // the whole S row into registers, then hand the TMEM columns back for S_{t+1}
      uint32_t sv[128];
      tmem_ld_32x32b_x32(tSrow + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld_32x32b_x32(tSrow + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld_32x32b_x32(tSrow + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
      tmem_ld_32x32b_x32(tSrow + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(s_free);
      // row maximum over four independent chains (a single chain of 128 dependent
      // maxima would cost its full latency per tile)
      float mx;
      {
        if (kvalid < kAK) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= kvalid) sv[i] = __float_as_uint(-INFINITY);
        }
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; i += 8) {
          m0 = max3(m0, __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
          m1 = max3(m1, __uint_as_float(sv[i + 2]), __uint_as_float(sv[i + 3]));
          m2 = max3(m2, __uint_as_float(sv[i + 4]), __uint_as_float(sv[i + 5]));
          m3 = max3(m3, __uint_as_float(sv[i + 6]), __uint_as_float(sv[i + 7]));
        }
        mx = max3(m0, m1, fmaxf(m2, m3));
      }
      // new running maximum; O is rescaled (after the wait below) only when it grew by more than 2^8
      float alpha = 1.f;
      bool rescale = false;
      if (first) {
        m_used = mx * sl2;
        l = 0.f;
      } else {
        const float m_new = fmaxf(m_used, mx * sl2);
        if (m_new > m_used + 8.f) {
          alpha = ex2(m_used - m_new);
          l *= alpha;
          m_used = m_new;
          rescale = true;
        }
      }
      // P = exp2(s*scale*log2e - m_used) as packed FP16 pairs in registers (masked keys give
      // exp2(-inf) = 0) while the previous PV product may still be running; the row sum in
      // four packed FP16 partial sums of 16 pairs each (every P <= 256, so no partial sum
      // exceeds 4096)
      uint32_t pk[64];
      uint32_t hs0 = 0u, hs1 = 0u, hs2 = 0u, hs3 = 0u;
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          float x0, x1;
          fma2(__uint_as_float(sv[2 * (i + u)]), __uint_as_float(sv[2 * (i + u) + 1]), sl2, -m_used, x0, x1);
          pk[i + u] = ex2_f16x2(cvt_f16x2(x0, x1));
        }
        hs0 = add_f16x2(hs0, pk[i]);
        hs1 = add_f16x2(hs1, pk[i + 1]);
        hs2 = add_f16x2(hs2, pk[i + 2]);
        hs3 = add_f16x2(hs3, pk[i + 3]);
      }
      // the previous PV product must be done before P is overwritten or O rescaled
      if (t > 0 && !mbar_wait_warp(pv_done, (t - 1) & 1, abort_flag, args.err)) break;
      tc_fence_after();
      // rows decide on their own whether O must be rescaled, but the TMEM round trip is
      // warp-collective: the warp makes it when any of its rows needs it, and the rows
      // that do not keep alpha = 1 (their O multiplied by 1, unchanged)
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tOrow + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st_32x32b_x32(tOrow + c * 32, r);
        }
        tmem_st_wait();
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        // keys c*32 .. c*32+31 = half c/2, 16-byte chunks 4*(c&1) .. +3, swizzled by row
        const uint32_t hrow = prow0 + (c >> 1) * kTileBytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c & 1) * 4 + q) ^ (row & 7);
          const int k = c * 16 + 4 * q;
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(hrow + chunk * 16), "r"(pk[k]),
                       "r"(pk[k + 1]), "r"(pk[k + 2]), "r"(pk[k + 3])
                       : "memory");
        }
      }
      l += (f16x2_sum(hs0) + f16x2_sum(hs1)) + (f16x2_sum(hs2) + f16x2_sum(hs3));
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
      if (!last) continue;

      // ---------------------------------------------------------- end of this CTA's part of item X
      if (!mbar_wait_warp(pv_done, t & 1, abort_flag, args.err)) break;
      tc_fence_after();
      {
        const int w_first = (int)cta_first_step(blockIdx.x, args.steps, args.ctas);  // recomputed: rarely needed
        attn_item_end(args, tOrow, row, (w_first + t) / nt, t >= j && j == nt - 1, (w_first + t) / nt == w_first / nt,
                      m_used, l);
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

// Merge of split items: block b looks at the boundary between CTAs b and b+1;
// if it falls inside an item and is that item's first boundary, the block
// merges the item's pieces in CTA order: M = max m_p, O = sum 2^(m_p - M) O_p /
// sum 2^(m_p - M) l_p. Four threads per query row, 16 output columns each; up to
// kMergeBatch pieces are loaded before any is used.
constexpr int kMergeBatch = 4;

__global__ void __launch_bounds__(512) attention_merge_kernel(const __grid_constant__ AttnArgs args) {
  pdl_wait();
  pdl_trigger();
  const int nt = args.ktiles;
  const int64_t b = blockIdx.x + 1;
  const int64_t s0 = cta_first_step(b, args.steps, args.ctas);
  if (s0 % nt == 0) return;  // boundary between items
  const int64_t sprev = cta_first_step(b - 1, args.steps, args.ctas);
  if (sprev / nt == s0 / nt && sprev % nt != 0) return;  // an earlier boundary merges this item
  const int X = (int)(s0 / nt);
  const int64_t s_hi = (int64_t)X * nt + nt - 1;
  const int64_t c_lo = b - 1;
  int64_t c_hi = b;
  while (c_hi + 1 < args.ctas && cta_first_step(c_hi + 1, args.steps, args.ctas) <= s_hi) ++c_hi;
  const int row = threadIdx.x >> 2, quarter = threadIdx.x & 3;
  float mmax = -INFINITY, lsum = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int64_t c0 = c_lo; c0 <= c_hi; c0 += kMergeBatch) {
    float m[kMergeBatch], l[kMergeBatch];
    float4 o[kMergeBatch][4];
#pragma unroll
    for (int p = 0; p < kMergeBatch; ++p) {
      const int64_t c = c0 + p;
      m[p] = -INFINITY;
      l[p] = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) o[p][u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c <= c_hi) {
        const int fi = (int)(cta_first_step(c, args.steps, args.ctas) / nt);
        const float* sl = args.partial + ((size_t)c * 2 + (X == fi ? 0 : 1)) * kSlotFloats;
        m[p] = __ldcg(sl + 8192 + row);
        l[p] = __ldcg(sl + 8320 + row);
        const float4* o4 = reinterpret_cast<const float4*>(sl + row * 64 + quarter * 16);
#pragma unroll
        for (int u = 0; u < 4; ++u) o[p][u] = __ldcg(o4 + u);
      }
    }
    float mb = mmax;
#pragma unroll
    for (int p = 0; p < kMergeBatch; ++p) mb = fmaxf(mb, m[p]);
    const float rescale = mmax == -INFINITY ? 0.f : ex2(mmax - mb);  // earlier batches to the new maximum
    lsum *= rescale;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= rescale;
#pragma unroll
    for (int p = 0; p < kMergeBatch; ++p) {
      const float e = m[p] == -INFINITY ? 0.f : ex2(m[p] - mb);
      lsum += e * l[p];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc[4 * u] += e * o[p][u].x;
        acc[4 * u + 1] += e * o[p][u].y;
        acc[4 * u + 2] += e * o[p][u].z;
        acc[4 * u + 3] += e * o[p][u].w;
      }
    }
    mmax = mb;
  }
  const int h = X / args.qtiles;
  const int qrow = (X % args.qtiles) * kAQ + row;
  if (qrow >= args.Nq) return;
  const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
  uint4* d4 = reinterpret_cast<uint4*>(args.O + (size_t)qrow * args.ldo + h * 64 + quarter * 16);
#pragma unroll
  for (int u = 0; u < 2; ++u)
    d4[u] = make_uint4(pack_bf16x2(acc[8 * u] * inv, acc[8 * u + 1] * inv),
                       pack_bf16x2(acc[8 * u + 2] * inv, acc[8 * u + 3] * inv),
                       pack_bf16x2(acc[8 * u + 4] * inv, acc[8 * u + 5] * inv),
                       pack_bf16x2(acc[8 * u + 6] * inv, acc[8 * u + 7] * inv));
}

size_t attention_partial_bytes(int num_sms) { return (size_t)2 * num_sms * 2 * kSlotFloats * sizeof(float); }

// Split the key tiles of items between CTAs only when that shortens the
// longest CTA: with whole items a CTA alone on its SM runs a step in about 0.6
// of the time two co-resident CTAs take; a split costs about ten steps (the
// extra Q loads and pipeline fills of the pieces and the merge kernel).
static bool attention_split_pays(int items, int ktiles, int num_sms) {
  if (ktiles < 2) return false;
  const int resident = 2 * num_sms;
  const double whole = items <= num_sms ? 0.6 * ktiles : (double)((items + resident - 1) / resident) * ktiles;
  const double split = (double)items * ktiles / resident + 10.0;
  return split < whole;
}

int attention_plan_launches(int Nq, int Nk, int heads, int num_sms) {
  const int items = heads * ((Nq + kAQ - 1) / kAQ);
  return attention_split_pays(items, (Nk + kAK - 1) / kAK, num_sms) ? 2 : 1;
}

int launch_attention_tc(const __nv_bfloat16* qbase, int q_ld, int q_rows, int q_col, const __nv_bfloat16* kvbase,
                        int kv_ld, int kv_rows, int k_col, int v_col, __nv_bfloat16* O, int ldo, int Nq, int Nk,
                        int heads, float* partial, size_t partial_bytes, int num_sms, int* err, cudaStream_t st) {
  if (Nq <= 0 || Nk <= 0 || heads <= 0) return 0;
  AttnMaps maps;
  memset(&maps, 0, sizeof(maps));
  if (!tmap_encode_2d(&maps.q, qbase, (uint64_t)q_ld, (uint64_t)q_rows, 64, 128)) return -2;
  if (!tmap_encode_2d(&maps.kv, kvbase, (uint64_t)kv_ld, (uint64_t)kv_rows, 64, 128)) return -2;
  AttnArgs a;
  a.Nq = Nq;
  a.Nk = Nk;
  a.q_col = q_col;
  a.k_col = k_col;
  a.v_col = v_col;
  a.O = O;
  a.ldo = ldo;
  a.scale_log2 = 0.125f * 1.4426950408889634f;
  a.qtiles = (Nq + kAQ - 1) / kAQ;
  a.ktiles = (Nk + kAK - 1) / kAK;
  const int items = heads * a.qtiles;
  a.steps = (int64_t)items * a.ktiles;
  const int resident = 2 * num_sms;
  const bool split = partial && partial_bytes >= attention_partial_bytes(num_sms) &&
                     attention_split_pays(items, a.ktiles, num_sms);
  // split: every CTA an equal share of the steps; otherwise one CTA per whole item
  a.ctas = split ? (int)std::min<int64_t>(resident, a.steps) : items;
  a.partial = partial;
  a.err = err;
  constexpr size_t smem = 1024 + 6 * kTileBytes + 128;
  static bool attr = false;  // benign race: identical value for every caller
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return (int)e;
    attr = true;
  }
  int e = (int)launch_pdl(attention_tc_kernel, dim3(a.ctas), dim3(192), smem, st, maps, a);
  if (e != 0 || !split || a.ctas < 2) return e;
  return (int)launch_pdl(attention_merge_kernel, dim3(a.ctas - 1), dim3(512), 0, st, a);
}

}  // namespace sdk
