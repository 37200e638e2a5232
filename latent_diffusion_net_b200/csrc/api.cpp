// C ABI of the library: argument validation, workspace planning and the launch
// sequences of the time embedding, conv_in, ResnetBlock2D, Transformer2DModel,
// downsample, upsample, output head and the whole denoiser step.
//
// Topology: "Stable Diffusion 2.1 Base 宏观架构" section 3 (Down 0-3 / Mid /
// Up 0-3 with skip connections) and "Stable Diffusion XL Inpainting 宏观架构"
// section 3; block composition: section 4 of both pages.
#include <cuda_runtime.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <utility>
#include <vector>

#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "profile.h"
#include "sd_api.h"
#include "weights.h"

using sdk::GemmProblem;
using namespace sdw;

namespace {

typedef __nv_bfloat16 bf16;

// ------------------------------------------------------------------ device cache
struct DevInfo {
  bool init = false;
  int sms = 148;
  int major = 0, minor = 0;
};
std::mutex g_dev_mu;
DevInfo g_dev[64];

sd_status device_info(DevInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return SD_ERR_LAUNCH;
  if (dev >= 64) return SD_ERR_UNSUPPORTED;  // the per-device cache holds 64 devices
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (!d.init) {
    if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return SD_ERR_LAUNCH;
    cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev);
    d.init = true;
  }
  *out = d;
  if (d.major != 10 || d.minor != 0) return SD_ERR_NOT_SM100;
  return SD_OK;
}

// ------------------------------------------------------------------ workspace arena
constexpr size_t kHeaderBytes = 256;   // word 0: device error flags
constexpr int kMaxGnLaunches = 128;      // GroupNorm statistics slots per call
constexpr int kMaxGroups = 64;
// per GroupNorm launch: one 128-byte line of sums per group, then a line holding
// the barrier counter of the single-pass kernel
constexpr int kGnSlotWords = sdk::kGnAccStride * kMaxGroups + 16;
constexpr size_t kGnAccBytes = (size_t)kMaxGnLaunches * kGnSlotWords * sizeof(unsigned long long);
constexpr int kMaxStatBlocks = 512;  // GroupNorm partial-sum slots: 2 CTAs per SM, up to 256 SMs


struct Arena {
  uint8_t* base;
  size_t off;
  void* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    void* p = base ? base + off : nullptr;
    off += bytes;
    return p;
  }
  bf16* bf(size_t elems) { return static_cast<bf16*>(take(elems * 2)); }
  float* f32(size_t elems) { return static_cast<float*>(take(elems * 4)); }
};

struct Ctx {
  cudaStream_t st;
  int* err;
  unsigned long long* gn_acc;  // [kMaxGnLaunches][kGnSlotWords], zeroed at the start of every call
  int* gn_seq;                 // host: GroupNorm launches issued so far in this call
  float* skws;  // split-K FP32 partial products
  size_t skws_bytes;
  float* attn_part;   // pieces of split attention items
  size_t attn_part_bytes;
  // two row-statistics buffers of [rs_rows][2] for the folded LayerNorms (zeroed every call);
  // *rs_clean is the host's record of the one that is zero now
  unsigned long long* rs[2];
  int64_t rs_rows;
  int* rs_clean;
  size_t clear_bytes;  // header, GroupNorm accumulators and row statistics: one memset per call
  int sms;
};

constexpr size_t kSplitKBytes = size_t(16) << 20;

// Header + GroupNorm scratch (+ row statistics for `rs_rows` tokens) at the start of every workspace.
Ctx make_ctx(Arena& ar, cudaStream_t st, int sms, int64_t rs_rows = 0) {
  Ctx c;
  const size_t rs_bytes = (size_t)rs_rows * 2 * sizeof(unsigned long long);
  c.clear_bytes = kHeaderBytes + kGnAccBytes + 2 * rs_bytes;
  uint8_t* h = static_cast<uint8_t*>(ar.take(c.clear_bytes));
  c.err = reinterpret_cast<int*>(h);
  c.gn_acc = h ? reinterpret_cast<unsigned long long*>(h + kHeaderBytes) : nullptr;
  c.rs_rows = rs_rows;
  c.rs[0] = h && rs_rows ? reinterpret_cast<unsigned long long*>(h + kHeaderBytes + kGnAccBytes) : nullptr;
  c.rs[1] = c.rs[0] ? c.rs[0] + rs_rows * 2 : nullptr;
  c.rs_clean = nullptr;
  c.gn_seq = nullptr;
  c.skws = static_cast<float*>(ar.take(kSplitKBytes));
  c.skws_bytes = kSplitKBytes;
  c.st = st;
  c.sms = sms < kMaxStatBlocks / 2 ? sms : kMaxStatBlocks / 2;
  c.attn_part_bytes = sdk::attention_partial_bytes(kMaxStatBlocks / 2);
  c.attn_part = static_cast<float*>(ar.take(c.attn_part_bytes));
  return c;
}

#define CK(x)                        \
  do {                               \
    int _e = (x);                    \
    if (_e == -1) return SD_ERR_UNSUPPORTED; \
    if (_e != 0) return SD_ERR_LAUNCH; \
  } while (0)

inline const bf16* W(const void* base, int64_t off) {
  return reinterpret_cast<const bf16*>(static_cast<const uint8_t*>(base) + off);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ------------------------------------------------------------------ building blocks

int run_gemv(const Ctx& c, const sdk::GemvBatch& b) {
  double rows = 0;
  for (int j = 0; j < b.njobs; ++j) rows += b.job[j].rows;
  sdp::Scope sc("gemv", sdp::F_GEMV, 2.0 * rows * b.K, 2.0 * rows * b.K, c.st);
  return sdk::launch_gemv(b, c.st);
}

// GroupNorm (+SiLU) of [x0 | x1] into y.
sd_status run_gn(const Ctx& c, const bf16* x0, int C0, const bf16* x1, int C1, int HW, int G, float eps,
                 const bf16* gamma, const bf16* beta, int silu, bf16* y) {
  if (!c.gn_seq || *c.gn_seq >= kMaxGnLaunches) return SD_ERR_UNSUPPORTED;
  unsigned long long* acc = c.gn_acc + (size_t)(*c.gn_seq)++ * kGnSlotWords;
  unsigned int* counter = reinterpret_cast<unsigned int*>(acc + sdk::kGnAccStride * kMaxGroups);
  const int nk = sdk::groupnorm_plan_launches(C0 + C1, HW, c.sms);
  // algorithmic bytes: read once and write once (the two-kernel form reads twice)
  sdp::Scope sc("groupnorm", sdp::F_GN_APPLY, 0, (nk == 1 ? 2.0 : 3.0) * HW * (C0 + C1) * 2, c.st, nk);
  CK(sdk::launch_groupnorm(x0, C0, x1, C1, HW, G, eps, gamma, beta, silu, y, acc, counter, c.sms, c.st, c.err));
  return SD_OK;
}

// Sublayer record (sd_record_*): per calling thread.
struct Recorder {
  bool on = false;
  uint8_t* buf = nullptr;
  size_t bytes = 0, used = 0;
  bool overflow = false;
  int res_count = 0, tx_count = 0;
  std::vector<sd_record_entry> entries;
};
thread_local Recorder t_rec;

// Device slot for one recorded [rows][cols] BF16 matrix, or null when it does not fit.
bf16* rec_slot(const char* name, int module, int block, int64_t rows, int64_t cols) {
  Recorder& r = t_rec;
  const size_t off = (r.used + 255) & ~size_t(255);
  const size_t need = (size_t)rows * cols * 2;
  if (off + need > r.bytes) {
    r.overflow = true;
    return nullptr;
  }
  sd_record_entry e;
  memset(&e, 0, sizeof(e));
  strncpy(e.name, name, sizeof(e.name) - 1);
  e.module = module;
  e.block = block;
  e.offset = (int64_t)off;
  e.rows = rows;
  e.cols = cols;
  r.entries.push_back(e);
  r.used = off + need;
  return reinterpret_cast<bf16*>(r.buf + off);
}

// Timeout injection for tests (sd_debug_inject_timeout).
std::atomic<int> g_inject_n{0}, g_inject_spins{0};

// Launch a GEMM problem under a profiling scope with its algorithmic work:
// FLOPs 2*M*N*K (K = reduction length; alg_k overrides a zero-padded K), bytes
// = every A source and B matrix read once, the output (and residual) once.
std::atomic<int> g_force_bn{0}, g_force_splits{0};

int launch_gemm(const Ctx& c, const GemmProblem& p0, double alg_k = 0) {
  GemmProblem p = p0;
  p.force_bn = g_force_bn.load(std::memory_order_relaxed);
  p.force_splits = g_force_splits.load(std::memory_order_relaxed);
  if (g_inject_n.load(std::memory_order_relaxed) > 0 && g_inject_n.fetch_sub(1) > 0)
    p.hold_spins = g_inject_spins.load(std::memory_order_relaxed);
  double K = 0;
  for (int i = 0; i < p.nseg; ++i) K += 64.0 * p.seg[i].nkb;
  if (alg_k > 0) K = alg_k;
  const double M = (double)p.Ho * p.Wo;
  const double fl = 2.0 * M * p.N * K;
  double by = 0;
  for (int i = 0; i < p.na; ++i) by += 2.0 * p.a[i].C * p.a[i].W * p.a[i].H * p.a[i].Z;
  for (int i = 0; i < p.nb; ++i) by += 2.0 * p.b[i].K * (p.b[i].rows < p.N ? p.b[i].rows : p.N);
  by += 2.0 * M * (p.epi.mode == sdk::GEMM_GEGLU ? p.N / 2 : p.N);
  if (p.epi.residual) by += 2.0 * M * p.N;
  sdp::Scope sc("gemm_tc", sdp::F_GEMM, fl, by, c.st, sdk::gemm_tc_plan_launches(p));
  return sdk::gemm_tc_launch(p, c.st);
}

GemmProblem base_problem(const Ctx& c) {
  GemmProblem p;
  memset(&p, 0, sizeof(p));
  p.err = c.err;
  p.splitk_ws = c.skws;
  p.splitk_ws_bytes = c.skws_bytes;
  return p;
}

void add_conv3x3_segs(GemmProblem& p, int amap, int bmap, int C) {
  for (int t = 0; t < 9; ++t) {
    sdk::GemmSeg& s = p.seg[p.nseg++];
    s.amap = amap;
    s.bmap = bmap;
    s.dx = t % 3 - 1;
    s.dy = t / 3 - 1;
    s.z = 0;
    s.c0 = 0;
    s.bk0 = t * C;
    s.nkb = C / 64;
  }
}

// y[M, N] = A[M, K] B[N, K]^T (+ epilogue), A a token matrix.
// LayerNorm folded into a linear layer. A producer GEMM adds its output rows'
// sums into `out` and zeroes `clear`; a consumer GEMM reads the raw LayerNorm
// input as A, its row sums from `in`, and the column terms c1 / c2 of B packed
// as W * gamma.
struct LnFold {
  unsigned long long* out = nullptr;
  unsigned long long* clear = nullptr;
  int64_t clear_elems = 0;
  const unsigned long long* in = nullptr;
  const float* c1 = nullptr;
  const float* c2 = nullptr;
  int cols = 0;
  float eps = 0.f;
};

sd_status run_linear(const Ctx& c, const bf16* A, int M, int K, const bf16* B, int N, const bf16* bias,
                     const bf16* residual, int ld_res, bf16* out, int ld_out, int mode = sdk::GEMM_PLAIN,
                     double alg_k = 0, const LnFold* ln = nullptr, int f16_begin = 0) {
  GemmProblem p = base_problem(c);
  p.Ho = 1;
  p.Wo = M;
  p.N = N;
  p.na = 1;
  p.a[0] = {A, K, M, 1, 1};
  p.nb = 1;
  p.b[0] = {B, K, N};
  p.nseg = 1;
  p.seg[0] = {0, 0, 0, 0, 0, 0, 0, K / 64};
  p.epi.bias = bias;
  p.epi.residual = residual;
  p.epi.ld_res = ld_res;
  p.epi.out = out;
  p.epi.ld_out = ld_out;
  p.epi.mode = mode;
  p.epi.f16_begin = f16_begin;
  if (ln) {
    p.epi.rowstat_out = ln->out;
    p.epi.rowstat_clear = ln->clear;
    p.epi.rowstat_clear_elems = ln->clear_elems;
    p.epi.rowstat_in = ln->in;
    p.epi.colscale = ln->c1;
    if (ln->in) p.epi.colvec = ln->c2;
    p.epi.ln_cols = ln->cols;
    p.epi.ln_eps = ln->eps;
  }
  CK(launch_gemm(c, p, alg_k));
  return SD_OK;
}

// 3x3 stride-1 convolution of a dense NHWC input (already normalised/activated).
sd_status run_conv3x3(const Ctx& c, const bf16* x, int H, int Wd, int C, const bf16* w, int N, const bf16* bias,
                      bf16* out) {
  GemmProblem p = base_problem(c);
  p.Ho = H;
  p.Wo = Wd;
  p.N = N;
  p.na = 1;
  p.a[0] = {x, C, Wd, H, 1};
  p.nb = 1;
  p.b[0] = {w, 9 * C, N};
  add_conv3x3_segs(p, 0, 0, C);
  p.epi.bias = bias;
  p.epi.out = out;
  p.epi.ld_out = N;
  CK(launch_gemm(c, p));
  return SD_OK;
}

// ResnetBlock2D given the per-channel time projection tproj (FP32 [c_out]).
// scratch: xn [HW, cin], h1 [HW, cout], hn [HW, cout].
struct ResScratch {
  bf16 *xn, *h1, *hn;
};
ResScratch plan_res_scratch(Arena& ar, int HW, int cin, int cout) {
  ResScratch s;
  s.xn = ar.bf((size_t)HW * cin);
  s.h1 = ar.bf((size_t)HW * cout);
  s.hn = ar.bf((size_t)HW * cout);
  return s;
}

sd_status run_resblock(const Ctx& c, const ResW& w, const void* pw, int H, int Wd, const bf16* x, int cx,
                       const bf16* skip, int cs, const float* tproj, int G, float eps, bf16* y, const ResScratch& s) {
  const int HW = H * Wd;
  const int cin = cx + cs;
  const int cout = w.c_out;
  const int rmod = t_rec.on ? t_rec.res_count++ : -1;
  sd_status r;
  if (rmod >= 0) {
    // the block input, so that h1 can be compared with a reference computed from the same input
    bf16* d = rec_slot("x_h1", rmod, 0, HW, cx);
    if (d && cudaMemcpyAsync(d, x, (size_t)HW * cx * 2, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return SD_ERR_LAUNCH;
    bf16* e = cs > 0 ? rec_slot("x_skip", rmod, 0, HW, cs) : nullptr;
    if (e && cudaMemcpyAsync(e, skip, (size_t)HW * cs * 2, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return SD_ERR_LAUNCH;
  }
  // h1 = conv1(SiLU(GN1([x | skip]))) + b1 + tproj
  if ((r = run_gn(c, x, cx, skip, cs, HW, G, eps, W(pw, w.n1g), W(pw, w.n1b), 1, s.xn)) != SD_OK) return r;
  {
    GemmProblem p = base_problem(c);
    p.Ho = H;
    p.Wo = Wd;
    p.N = cout;
    p.na = 1;
    p.a[0] = {s.xn, cin, Wd, H, 1};
    p.nb = 1;
    p.b[0] = {W(pw, w.c1w), 9 * cin, cout};
    add_conv3x3_segs(p, 0, 0, cin);
    p.epi.bias = W(pw, w.c1b);
    p.epi.colvec = tproj;
    p.epi.out = s.h1;
    p.epi.ld_out = cout;
    CK(launch_gemm(c, p));
  }
  if (rmod >= 0) {
    bf16* d = rec_slot("h1", rmod, 0, HW, cout);
    if (d && cudaMemcpyAsync(d, s.h1, (size_t)HW * cout * 2, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return SD_ERR_LAUNCH;
  }
  // y = conv2(SiLU(GN2(h1))) + b2 + shortcut
  if ((r = run_gn(c, s.h1, cout, nullptr, 0, HW, G, eps, W(pw, w.n2g), W(pw, w.n2b), 1, s.hn)) != SD_OK) return r;
  {
    GemmProblem p = base_problem(c);
    p.Ho = H;
    p.Wo = Wd;
    p.N = cout;
    p.na = 1;
    p.a[0] = {s.hn, cout, Wd, H, 1};
    p.nb = 1;
    p.b[0] = {W(pw, w.c2w), 9 * cout, cout};
    add_conv3x3_segs(p, 0, 0, cout);
    p.epi.bias = W(pw, w.c2b);
    p.epi.out = y;
    p.epi.ld_out = cout;
    if (w.sw >= 0) {
      // 1x1 shortcut over [x | skip] as extra K-segments of the same accumulator
      p.a[1] = {x, cx, Wd, H, 1};
      p.na = 2;
      p.nb = 2;
      p.b[1] = {W(pw, w.sw), cin, cout};
      p.seg[p.nseg++] = {1, 1, 0, 0, 0, 0, 0, cx / 64};
      if (cs > 0) {
        p.a[2] = {skip, cs, Wd, H, 1};
        p.na = 3;
        p.seg[p.nseg++] = {2, 1, 0, 0, 0, 0, cx, cs / 64};
      }
      p.epi.bias2 = W(pw, w.sb);
    } else {
      p.epi.residual = x;
      p.epi.ld_res = cout;
    }
    CK(launch_gemm(c, p));
  }
  return SD_OK;
}

struct TxScratch {
  bf16 *nrm, *t, *ao, *big, *kv;
};
TxScratch plan_tx_scratch(Arena& ar, int HW, int C, int ctx_len) {
  TxScratch s;
  s.nrm = ar.bf((size_t)HW * C);
  s.t = ar.bf((size_t)HW * C);
  s.ao = ar.bf((size_t)HW * C);
  s.big = ar.bf((size_t)HW * 4 * C);
  s.kv = ar.bf((size_t)ctx_len * 2 * C);
  return s;
}

// Attention of Q (rows of qbase, columns q_col + 64h) against K/V (rows of
// kvbase, columns k_col + 64h and v_col + 64h), head_dim 64, into O [Nq, ldo].
int run_attn(const Ctx& c, const bf16* qbase, int q_ld, int q_col, const bf16* kvbase, int kv_ld, int k_col,
             int v_col, bf16* o, int ldo, int Nq, int Nk, int heads) {
  const double C = 64.0 * heads;
  sdp::Scope sc("attention", sdp::F_ATTN, 4.0 * Nq * Nk * C, 2.0 * C * (2.0 * Nq + 2.0 * Nk), c.st,
                sdk::attention_plan_launches(Nq, Nk, heads, c.sms));
  return sdk::launch_attention_tc(qbase, q_ld, Nq, q_col, kvbase, kv_ld, Nk, k_col, v_col, o, ldo, Nq, Nk, heads,
                                  c.attn_part, c.attn_part_bytes, c.sms, c.err, c.st);
}

// Transformer2DModel; y may alias x.
// The context K/V of every cross-attention of a model, projected by one GEMM at
// the start of the step: [ctx_len, ld] with the K columns of all blocks first and
// their V columns (FP16) from v_begin on; block b reads K at b.ctx_k_col.
struct CtxKV {
  const bf16* kv;
  int ld, v_begin;
};

sd_status run_transformer(const Ctx& c, const TxW& w, const void* pw, int H, int Wd, const bf16* x, const bf16* ctx,
                          int ctx_len, int G, float gn_eps, float ln_eps, bf16* y, const TxScratch& s,
                          const CtxKV* pre = nullptr) {
  const int HW = H * Wd;
  const int C = w.C;
  const int heads = C / 64;
  if (!c.rs[0] || !c.rs_clean || c.rs_rows < HW) return SD_ERR_UNSUPPORTED;
  const int tmod = t_rec.on ? t_rec.tx_count++ : -1;
  int bi = 0;  // BasicTransformer block index
  // recorded sublayer output before its residual add: the same linear layer without the residual
  auto record = [&](const char* name, const bf16* A, int K, int64_t w_off, int64_t b_off) -> sd_status {
    if (tmod < 0) return SD_OK;
    bf16* d = rec_slot(name, tmod, bi, HW, C);
    if (!d) return SD_OK;
    return run_linear(c, A, HW, K, W(pw, w_off), C, W(pw, b_off), nullptr, 0, d, C);
  };
  // the residual stream entering a sublayer (the sublayer's input before its LayerNorm)
  auto record_in = [&](const char* name) -> sd_status {
    if (tmod < 0) return SD_OK;
    bf16* d = rec_slot(name, tmod, bi, HW, C);
    if (d && cudaMemcpyAsync(d, s.t, (size_t)HW * C * 2, cudaMemcpyDeviceToDevice, c.st) != cudaSuccess)
      return SD_ERR_LAUNCH;
    return SD_OK;
  };
  // The three LayerNorms of each block are folded into the GEMMs they feed
  // (Q/K/V, the cross-attention query, FF1): every GEMM that writes the
  // residual stream t also leaves t's row sums in one of two buffers, and
  // zeroes the other one, whose last reader ran before it.
  int cur = -1;              // buffer holding the row sums of t
  int clean = *c.rs_clean;  // buffer that is zero
  auto producer = [&]() {
    LnFold f;
    f.out = c.rs[clean];
    f.clear = cur >= 0 ? c.rs[cur] : nullptr;
    f.clear_elems = c.rs_rows * 2;
    if (cur >= 0) {
      std::swap(cur, clean);
    } else {
      cur = clean;
      clean = 1 - clean;
    }
    return f;
  };
  auto consumer = [&](int64_t c1, int64_t c2) {
    LnFold f;
    f.in = c.rs[cur];
    f.c1 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(pw) + c1);
    f.c2 = reinterpret_cast<const float*>(static_cast<const uint8_t*>(pw) + c2);
    f.cols = C;
    f.eps = ln_eps;
    return f;
  };
  sd_status r;
  if ((r = run_gn(c, x, C, nullptr, 0, HW, G, gn_eps, W(pw, w.ng), W(pw, w.nb), 0, s.nrm)) != SD_OK) return r;
  {
    // the other buffer is not known to be zero yet: clear it too
    LnFold f = producer();
    f.clear = c.rs[clean];
    if ((r = run_linear(c, s.nrm, HW, C, W(pw, w.piw), C, W(pw, w.pib), nullptr, 0, s.t, C, sdk::GEMM_PLAIN, 0,
                        &f)) != SD_OK)
      return r;
  }
  for (const TxBlockW& b : w.blocks) {
    // self-attention: t += Wo Attn(LN1(t)), LN1 folded into the Q/K/V GEMM
    if ((r = record_in("x_attn1")) != SD_OK) return r;
    {
      const LnFold f = consumer(b.qkv_c1, b.qkv_c2);
      // V (columns 2C..3C) is stored as FP16: the attention kernel multiplies it with FP16 probabilities
      if ((r = run_linear(c, s.t, HW, C, W(pw, b.qkv), 3 * C, nullptr, nullptr, 0, s.big, 3 * C, sdk::GEMM_PLAIN, 0,
                          &f, 2 * C)) != SD_OK)
        return r;
    }
    CK(run_attn(c, s.big, 3 * C, 0, s.big, 3 * C, C, 2 * C, s.ao, C, HW, HW, heads));
    if ((r = record("attn1", s.ao, C, b.o1w, b.o1b)) != SD_OK) return r;
    {
      const LnFold f = producer();
      if ((r = run_linear(c, s.ao, HW, C, W(pw, b.o1w), C, W(pw, b.o1b), s.t, C, s.t, C, sdk::GEMM_PLAIN, 0,
                          &f)) != SD_OK)
        return r;
    }
    // cross-attention: t += Wo' Attn(LN2(t), ctx)
    if ((r = record_in("x_attn2")) != SD_OK) return r;
    {
      const LnFold f = consumer(b.q2_c1, b.q2_c2);
      if ((r = run_linear(c, s.t, HW, C, W(pw, b.q2), C, nullptr, nullptr, 0, s.big, C, sdk::GEMM_PLAIN, 0, &f)) !=
          SD_OK)
        return r;
    }
    if (b.kv2 >= 0) {
      if ((r = run_linear(c, ctx, ctx_len, w.ctx_dim, W(pw, b.kv2), 2 * C, nullptr, nullptr, 0, s.kv, 2 * C,
                          sdk::GEMM_PLAIN, 0, nullptr, C)) != SD_OK)  // V as FP16
        return r;
      CK(run_attn(c, s.big, C, 0, s.kv, 2 * C, 0, C, s.ao, C, HW, ctx_len, heads));
    } else {
      if (!pre || b.ctx_k_col < 0) return SD_ERR_UNSUPPORTED;
      CK(run_attn(c, s.big, C, 0, pre->kv, pre->ld, b.ctx_k_col, pre->v_begin + b.ctx_k_col, s.ao, C, HW, ctx_len,
                  heads));
    }
    if ((r = record("attn2", s.ao, C, b.o2w, b.o2b)) != SD_OK) return r;
    {
      const LnFold f = producer();
      if ((r = run_linear(c, s.ao, HW, C, W(pw, b.o2w), C, W(pw, b.o2b), s.t, C, s.t, C, sdk::GEMM_PLAIN, 0,
                          &f)) != SD_OK)
        return r;
    }
    // GEGLU feed-forward: t += W2 (a * GELU(g)) + b2, LN3 folded into FF1 (its bias is in c2)
    if ((r = record_in("x_ff")) != SD_OK) return r;
    {
      const LnFold f = consumer(b.f1_c1, b.f1_c2);
      if ((r = run_linear(c, s.t, HW, C, W(pw, b.f1w), 8 * C, nullptr, nullptr, 0, s.big, 4 * C, sdk::GEMM_GEGLU, 0,
                          &f)) != SD_OK)
        return r;
    }
    if ((r = record("ff", s.big, 4 * C, b.f2w, b.f2b)) != SD_OK) return r;
    {
      const LnFold f = producer();
      if ((r = run_linear(c, s.big, HW, 4 * C, W(pw, b.f2w), C, W(pw, b.f2b), s.t, C, s.t, C, sdk::GEMM_PLAIN, 0,
                          &f)) != SD_OK)
        return r;
    }
    ++bi;
  }
  *c.rs_clean = clean;
  // y = x + proj_out(t)
  return run_linear(c, s.t, HW, C, W(pw, w.pow_), C, W(pw, w.pob), x, C, y, C);
}

sd_status run_downsample(const Ctx& c, const ConvW& w, const void* pw, int H, int Wd, int C, const bf16* x, bf16* y,
                         bf16* planes) {
  const int Ho = H / 2, Wo = Wd / 2;
  {
    sdp::Scope sc("phase_split", sdp::F_OTHER, 0, 4.0 * H * Wd * C, c.st);
    CK(sdk::launch_phase_split(x, H, Wd, C, planes, c.st));
  }
  GemmProblem p = base_problem(c);
  p.Ho = Ho;
  p.Wo = Wo;
  p.N = C;
  p.na = 1;
  p.a[0] = {planes, C, Wo, Ho, 4};
  p.nb = 1;
  p.b[0] = {W(pw, w.w), 9 * C, C};
  for (int t = 0; t < 9; ++t) {
    const int r = t / 3, q = t % 3;
    sdk::GemmSeg& s = p.seg[p.nseg++];
    s.amap = 0;
    s.bmap = 0;
    s.dy = r == 0 ? -1 : 0;
    s.dx = q == 0 ? -1 : 0;
    s.z = (r == 1 ? 0 : 2) + (q == 1 ? 0 : 1);
    s.c0 = 0;
    s.bk0 = t * C;
    s.nkb = C / 64;
  }
  p.epi.bias = W(pw, w.b);
  p.epi.out = y;
  p.epi.ld_out = C;
  CK(launch_gemm(c, p));
  return SD_OK;
}

sd_status run_upsample(const Ctx& c, const ConvW& w, const void* pw, int H, int Wd, int C, const bf16* x, bf16* y,
                       bf16* up) {
  {
    sdp::Scope sc("upsample2x", sdp::F_OTHER, 0, 10.0 * H * Wd * C, c.st);
    CK(sdk::launch_upsample2x(x, H, Wd, C, up, c.st));
  }
  return run_conv3x3(c, up, 2 * H, 2 * Wd, C, W(pw, w.w), C, W(pw, w.b), y);
}

sd_status run_conv_in(const Ctx& c, const ConvW& w, const void* pw, int kp, int H, int Wd, const bf16* s0, int c0,
                      const bf16* s1, int c1, const bf16* s2, int c2, int cout, bf16* y, bf16* col) {
  {
    sdp::Scope sc("conv_in_im2col", sdp::F_OTHER, 0, 2.0 * H * Wd * (c0 + c1 + c2 + kp), c.st);
    CK(sdk::launch_conv_in_im2col(s0, c0, s1, c1, s2, c2, H, Wd, kp, col, c.st));
  }
  return run_linear(c, col, H * Wd, kp, W(pw, w.w), cout, W(pw, w.b), nullptr, 0, y, cout, sdk::GEMM_PLAIN,
                    9.0 * (c0 + c1 + c2));
}

sd_status run_output(const Ctx& c, const OutW& w, const void* pw, int H, int Wd, int C, int cout, int G, float eps,
                     const bf16* x, bf16* y, bf16* xn) {
  sd_status r = run_gn(c, x, C, nullptr, 0, H * Wd, G, eps, W(pw, w.ng), W(pw, w.nb), 1, xn);
  if (r != SD_OK) return r;
  return run_conv3x3(c, xn, H, Wd, C, W(pw, w.w), cout, W(pw, w.b), y);
}

sd_status run_time(const Ctx& c, const TimeW& w, const void* pw, int proj, int temb_dim, float t, float* phi,
                   float* hid, float* temb) {
  {
    sdp::Scope sc("sinusoid", sdp::F_OTHER, 0, 4.0 * proj, c.st);
    CK(sdk::launch_sinusoid(t, proj, phi, c.st));
  }
  sdk::GemvBatch b;
  memset(&b, 0, sizeof(b));
  b.njobs = 1;
  b.K = proj;
  b.silu_out = 1;
  b.x = phi;
  b.job[0] = {W(pw, w.l1w), W(pw, w.l1b), hid, temb_dim};
  CK(run_gemv(c, b));
  b.K = temb_dim;
  b.silu_out = 0;
  b.x = hid;
  b.job[0] = {W(pw, w.l2w), W(pw, w.l2b), temb, temb_dim};
  CK(run_gemv(c, b));
  return SD_OK;
}

// Single-head self-attention of the VAE MidBlock over the H*W tokens:
// y = x + (softmax(Q K^T / sqrt(C)) V) W_o^T + b_o with Q, K, V from GN(x). The
// head is C = 512 wide, so the scores are formed explicitly: an FP32 [HW, HW]
// score GEMM (Q against the K columns of the same matrix), a row softmax to
// BF16 probabilities, V transposed once, and the probability GEMM.
struct VaeAttnScratch {
  bf16 *nrm, *qkv, *vt, *o, *p;
  float* s;
};
VaeAttnScratch plan_vae_attn_scratch(Arena& ar, int64_t HW, int C) {
  VaeAttnScratch v;
  v.nrm = ar.bf((size_t)HW * C);
  v.qkv = ar.bf((size_t)HW * 3 * C);
  v.vt = ar.bf((size_t)HW * C);
  v.o = ar.bf((size_t)HW * C);
  v.p = ar.bf((size_t)HW * HW);
  v.s = ar.f32((size_t)HW * HW);
  return v;
}

sd_status run_vae_attention(const Ctx& c, const VaeAttnW& w, const void* pw, int H, int Wd, int G, float eps,
                            const bf16* x, bf16* y, const VaeAttnScratch& s) {
  const int HW = H * Wd;
  const int C = w.C;
  sd_status r;
  if ((r = run_gn(c, x, C, nullptr, 0, HW, G, eps, W(pw, w.ng), W(pw, w.nb), 0, s.nrm)) != SD_OK) return r;
  if ((r = run_linear(c, s.nrm, HW, C, W(pw, w.qkv), 3 * C, W(pw, w.qkv_b), nullptr, 0, s.qkv, 3 * C)) != SD_OK)
    return r;
  {
    // S = Q K^T: A = the Q columns of qkv, B = the K columns of the same matrix (rows = keys)
    GemmProblem p = base_problem(c);
    p.Ho = 1;
    p.Wo = HW;
    p.N = HW;
    p.na = 1;
    p.a[0] = {s.qkv, 3 * C, HW, 1, 1};
    p.nb = 1;
    p.b[0] = {s.qkv, 3 * C, HW};
    p.nseg = 1;
    p.seg[0] = {0, 0, 0, 0, 0, 0, C, C / 64};
    p.epi.out = reinterpret_cast<bf16*>(s.s);
    p.epi.ld_out = HW;
    p.epi.mode = sdk::GEMM_F32;
    CK(launch_gemm(c, p));
  }
  {
    sdp::Scope sc("softmax_rows", sdp::F_OTHER, 0, (double)HW * HW * 6.0, c.st);
    CK(sdk::launch_softmax_rows(s.s, HW, HW, HW, 1.0f / sqrtf((float)C), s.p, HW, c.st));
  }
  {
    sdp::Scope sc("transpose", sdp::F_OTHER, 0, 4.0 * HW * C, c.st);
    CK(sdk::launch_transpose(s.qkv, 3 * C, 2 * C, HW, C, s.vt, HW, c.st));
  }
  if ((r = run_linear(c, s.p, HW, HW, s.vt, C, nullptr, nullptr, 0, s.o, C)) != SD_OK) return r;
  return run_linear(c, s.o, HW, C, W(pw, w.ow), C, W(pw, w.ob), x, C, y, C);
}

// ------------------------------------------------------------------ validation helpers
bool ch_ok(int c) { return c > 0 && c % 64 == 0; }
bool groups_ok(int C, int G) { return G > 0 && G <= kMaxGroups && C % G == 0 && C / G >= 8; }

sd_status check_res(const sd_resblock_cfg* cfg) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->batch != 1) return SD_ERR_UNSUPPORTED;
  if (cfg->height <= 0 || cfg->width <= 0 || cfg->temb_dim <= 0 || cfg->temb_dim % 8) return SD_ERR_BAD_SHAPE;
  if (!ch_ok(cfg->c_x) || !ch_ok(cfg->c_out) || cfg->c_skip < 0 || cfg->c_skip % 64) return SD_ERR_UNSUPPORTED;
  if (!groups_ok(cfg->c_x + cfg->c_skip, cfg->groups) || !groups_ok(cfg->c_out, cfg->groups)) return SD_ERR_UNSUPPORTED;
  if (cfg->c_x + cfg->c_skip > 8192 || cfg->c_out > 8192) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

sd_status check_tx(const sd_transformer_cfg* cfg) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->batch != 1 || cfg->head_dim != 64) return SD_ERR_UNSUPPORTED;
  if (cfg->height <= 0 || cfg->width <= 0 || cfg->depth <= 0 || cfg->ctx_len <= 0) return SD_ERR_BAD_SHAPE;
  if (!ch_ok(cfg->channels) || cfg->channels > 2048 || !ch_ok(cfg->ctx_dim)) return SD_ERR_UNSUPPORTED;
  if (!groups_ok(cfg->channels, cfg->groups)) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

sd_status check_time(const sd_time_cfg* cfg) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->proj_dim <= 0 || cfg->proj_dim % 16 || cfg->temb_dim <= 0 || cfg->temb_dim % 8) return SD_ERR_BAD_SHAPE;
  return SD_OK;
}

sd_status check_conv(const sd_conv_cfg* cfg, int kind) {
  if (!cfg) return SD_ERR_NULL_ARG;
  if (cfg->batch != 1) return SD_ERR_UNSUPPORTED;
  if (cfg->height <= 0 || cfg->width <= 0) return SD_ERR_BAD_SHAPE;
  switch (kind) {
    case SD_CONV_IN:
      if (cfg->c_in != 4 && cfg->c_in != 9) return SD_ERR_UNSUPPORTED;
      if (!ch_ok(cfg->c_out)) return SD_ERR_UNSUPPORTED;
      return SD_OK;
    case SD_CONV_DOWNSAMPLE:
      if (cfg->height % 2 || cfg->width % 2) return SD_ERR_BAD_SHAPE;
      /* fallthrough */
    case SD_CONV_UPSAMPLE:
      if (!ch_ok(cfg->c_in) || cfg->c_out != cfg->c_in) return SD_ERR_UNSUPPORTED;
      return SD_OK;
    case SD_CONV_OUTPUT:
      if (!ch_ok(cfg->c_in) || cfg->c_out <= 0 || cfg->c_out > 16) return SD_ERR_UNSUPPORTED;
      if (!groups_ok(cfg->c_in, cfg->groups)) return SD_ERR_UNSUPPORTED;
      return SD_OK;
    default:
      return SD_ERR_UNSUPPORTED;
  }
}

sd_status check_unet(const sd_unet_cfg* cfg) {
  if (!cfg) return SD_ERR_NULL_ARG;
  const int L = cfg->n_levels;
  if (L < 1 || L > 4) return SD_ERR_UNSUPPORTED;
  if (cfg->in_channels != 4 && cfg->in_channels != 9) return SD_ERR_UNSUPPORTED;
  if (cfg->out_channels <= 0 || cfg->out_channels > 16) return SD_ERR_UNSUPPORTED;
  if (cfg->head_dim != 64 || cfg->layers_per_block < 1 || cfg->mid_depth < 1) return SD_ERR_UNSUPPORTED;
  const int div = 1 << (L - 1);
  if (cfg->height <= 0 || cfg->width <= 0 || cfg->height % div || cfg->width % div) return SD_ERR_BAD_SHAPE;
  if (cfg->ctx_len <= 0 || !ch_ok(cfg->ctx_dim)) return SD_ERR_BAD_SHAPE;
  if (cfg->time_proj_dim <= 0 || cfg->time_proj_dim % 16 || cfg->temb_dim <= 0 || cfg->temb_dim % 8)
    return SD_ERR_BAD_SHAPE;
  if (cfg->layers_per_block + 1 > 8) return SD_ERR_UNSUPPORTED;
  if (cfg->add_text_dim < 0 || cfg->add_time_ids < 0 || cfg->add_time_ids > sdk::kMaxAddIds) return SD_ERR_UNSUPPORTED;
  if (cfg->add_text_dim > 0) {
    if (cfg->add_time_ids > 0 && (cfg->add_time_dim <= 0 || cfg->add_time_dim % 2)) return SD_ERR_BAD_SHAPE;
    const int d = cfg->add_text_dim + cfg->add_time_ids * cfg->add_time_dim;
    if (d % 8 || d > 16384) return SD_ERR_UNSUPPORTED;  // 16-byte weight rows in the GEMV; x staged in shared memory
  }
  for (int l = 0; l < L; ++l) {
    if (!ch_ok(cfg->block_channels[l]) || cfg->block_channels[l] > 2048) return SD_ERR_UNSUPPORTED;
    if (!groups_ok(cfg->block_channels[l], cfg->groups) || cfg->attn_depth[l] < 0) return SD_ERR_UNSUPPORTED;
  }
  return SD_OK;
}

sd_status check_vae(const sd_vae_cfg* cfg) {
  if (!cfg) return SD_ERR_NULL_ARG;
  const int L = cfg->n_levels;
  if (L < 1 || L > 4 || cfg->layers_per_block < 0 || cfg->layers_per_block > 7) return SD_ERR_UNSUPPORTED;
  if (cfg->latent_channels < 1 || cfg->latent_channels > 16 || cfg->out_channels < 1 || cfg->out_channels > 16)
    return SD_ERR_UNSUPPORTED;
  if (cfg->height <= 0 || cfg->width <= 0) return SD_ERR_BAD_SHAPE;
  if ((cfg->height * cfg->width) % 64) return SD_ERR_UNSUPPORTED;  // the attention's token count is a K dimension
  if (!(cfg->scaling_factor > 0.f)) return SD_ERR_BAD_SHAPE;
  for (int l = 0; l < L; ++l) {
    const int C = cfg->block_channels[l];
    if (!ch_ok(C) || C > 2048) return SD_ERR_UNSUPPORTED;
    // GroupNorm: at least 8 channels per group, or exactly 4 (an 8-channel vector then covers two whole groups)
    const int G = cfg->groups;
    if (G <= 0 || G > kMaxGroups || C % G || (C / G < 8 && C / G != 4)) return SD_ERR_UNSUPPORTED;
  }
  // the full score matrix of the MidBlock attention lives in the workspace (FP32 + BF16)
  const int64_t hw = (int64_t)cfg->height * cfg->width;
  if (hw > 16384 * 4) return SD_ERR_UNSUPPORTED;
  return SD_OK;
}

// ------------------------------------------------------------------ per-module workspace plans
struct ResPlan {
  Ctx c;
  ResScratch s;
  float* tproj;
};
size_t plan_res(Arena& ar, const sd_resblock_cfg* cfg, cudaStream_t st, int sms, ResPlan* p) {
  const int HW = cfg->height * cfg->width;
  p->c = make_ctx(ar, st, sms);
  p->tproj = ar.f32(cfg->c_out);
  p->s = plan_res_scratch(ar, HW, cfg->c_x + cfg->c_skip, cfg->c_out);
  return ar.off;
}

struct TxPlan {
  Ctx c;
  TxScratch s;
};
size_t plan_tx(Arena& ar, const sd_transformer_cfg* cfg, cudaStream_t st, int sms, TxPlan* p) {
  p->c = make_ctx(ar, st, sms, (int64_t)cfg->height * cfg->width);
  p->s = plan_tx_scratch(ar, cfg->height * cfg->width, cfg->channels, cfg->ctx_len);
  return ar.off;
}

struct ConvPlan {
  Ctx c;
  bf16* scratch;
};
size_t plan_conv(Arena& ar, const sd_conv_cfg* cfg, int kind, cudaStream_t st, int sms, ConvPlan* p) {
  const size_t HW = (size_t)cfg->height * cfg->width;
  p->c = make_ctx(ar, st, sms);
  switch (kind) {
    case SD_CONV_IN: p->scratch = ar.bf(HW * conv_in_kp(cfg->c_in)); break;
    case SD_CONV_DOWNSAMPLE: p->scratch = ar.bf(HW * cfg->c_in); break;
    case SD_CONV_UPSAMPLE: p->scratch = ar.bf(4 * HW * cfg->c_in); break;
    default: p->scratch = ar.bf(HW * cfg->c_in); break;
  }
  return ar.off;
}

struct TimePlan {
  Ctx c;
  float *phi, *hid;
};
size_t plan_time(Arena& ar, const sd_time_cfg* cfg, cudaStream_t st, int sms, TimePlan* p) {
  p->c = make_ctx(ar, st, sms);
  p->phi = ar.f32(cfg->proj_dim);
  p->hid = ar.f32(cfg->temb_dim);
  return ar.off;
}

// Whole step.
struct UNetPlan {
  Ctx c;
  float *phi, *hid, *temb, *tproj;
  float *add_x, *add_h;  // SDXL added conditioning: MLP input and hidden layer
  std::vector<bf16*> skip;      // 1 + L*lpb + (L-1) slots, push order
  std::vector<int> skip_c, skip_hw;
  bf16 *pp[2];                  // up-path ping-pong
  ResScratch rs;
  TxScratch ts;
  bf16* conv_scratch;
  bf16 *mid_a, *mid_b;
  bf16* ctx_kv;     // [ctx_len, 2 * ctx_k_cols]: the context K/V of every cross-attention
  int ctx_k_cols;
};

size_t plan_unet(Arena& ar, const sd_unet_cfg* cfg, cudaStream_t st, int sms, UNetPlan* p) {
  const int L = cfg->n_levels;
  const int* ch = cfg->block_channels;
  p->c = make_ctx(ar, st, sms, (int64_t)cfg->height * cfg->width);  // the largest level
  p->phi = ar.f32(cfg->time_proj_dim);
  p->hid = ar.f32(cfg->temb_dim);
  p->temb = ar.f32(cfg->temb_dim);
  p->add_x = p->add_h = nullptr;
  if (cfg->add_text_dim > 0) {
    p->add_x = ar.f32((size_t)cfg->add_text_dim + (size_t)cfg->add_time_ids * cfg->add_time_dim);
    p->add_h = ar.f32(cfg->temb_dim);
  }
  // K width of the context K/V matrix: C per BasicTransformer block of every cross-attention
  int kcols = cfg->mid_depth * ch[L - 1];
  for (int l = 0; l < L; ++l)
    if (cfg->attn_depth[l] > 0) kcols += (2 * cfg->layers_per_block + 1) * cfg->attn_depth[l] * ch[l];
  p->ctx_k_cols = kcols;
  p->ctx_kv = ar.bf((size_t)cfg->ctx_len * 2 * kcols);
  int64_t tsum = 0;
  for (int l = 0; l < L; ++l) tsum += (int64_t)ch[l] * (2 * cfg->layers_per_block + 1);
  tsum += 2 * ch[L - 1];
  p->tproj = ar.f32((size_t)tsum);
  // skip slots
  int H = cfg->height, Wd = cfg->width;
  p->skip.clear();
  p->skip_c.clear();
  p->skip_hw.clear();
  auto push = [&](int c, int hw) {
    p->skip.push_back(ar.bf((size_t)hw * c));
    p->skip_c.push_back(c);
    p->skip_hw.push_back(hw);
  };
  push(ch[0], H * Wd);
  size_t max_res = 0, max_tx = 0, max_conv = 0;
  auto res_need = [&](int hw, int cin, int cout) {
    size_t n = ((size_t)hw * cin * 2 + 255) / 256 * 256 + 2 * (((size_t)hw * cout * 2 + 255) / 256 * 256);
    if (n > max_res) max_res = n;
  };
  auto tx_need = [&](int hw, int C) {
    size_t n = 7 * (((size_t)hw * C * 2 + 255) / 256 * 256) + (size_t)cfg->ctx_len * 2 * C * 2 + 1024;
    if (n > max_tx) max_tx = n;
  };
  size_t conv_need = (size_t)cfg->height * cfg->width * conv_in_kp(cfg->in_channels) * 2;
  max_conv = conv_need;
  int c_prev = ch[0];
  for (int l = 0; l < L; ++l) {
    for (int i = 0; i < cfg->layers_per_block; ++i) {
      res_need(H * Wd, c_prev, ch[l]);
      c_prev = ch[l];
      if (cfg->attn_depth[l] > 0) tx_need(H * Wd, ch[l]);
      push(ch[l], H * Wd);
    }
    if (l < L - 1) {
      if ((size_t)H * Wd * ch[l] * 2 > max_conv) max_conv = (size_t)H * Wd * ch[l] * 2;  // phase planes
      H /= 2;
      Wd /= 2;
      push(ch[l], H * Wd);
    }
  }
  res_need(H * Wd, ch[L - 1], ch[L - 1]);
  tx_need(H * Wd, ch[L - 1]);
  p->mid_a = ar.bf((size_t)H * Wd * ch[L - 1]);
  p->mid_b = ar.bf((size_t)H * Wd * ch[L - 1]);
  // up path
  size_t max_pp = 0;
  std::vector<int> sc = p->skip_c;
  c_prev = ch[L - 1];
  for (int up = 0; up < L; ++up) {
    const int l = L - 1 - up;
    for (int i = 0; i <= cfg->layers_per_block; ++i) {
      const int cs = sc.back();
      sc.pop_back();
      res_need(H * Wd, c_prev + cs, ch[l]);
      c_prev = ch[l];
      if (cfg->attn_depth[l] > 0) tx_need(H * Wd, ch[l]);
      if ((size_t)H * Wd * ch[l] > max_pp) max_pp = (size_t)H * Wd * ch[l];
    }
    if (up < L - 1) {
      const size_t upsz = (size_t)4 * H * Wd * ch[l] * 2;  // materialised nearest-2x input
      if (upsz > max_conv) max_conv = upsz;
      H *= 2;
      Wd *= 2;
      if ((size_t)H * Wd * ch[l] > max_pp) max_pp = (size_t)H * Wd * ch[l];
    }
  }
  // output head GN scratch
  if ((size_t)H * Wd * ch[0] * 2 > max_conv) max_conv = (size_t)H * Wd * ch[0] * 2;
  p->pp[0] = ar.bf(max_pp);
  p->pp[1] = ar.bf(max_pp);
  // shared module scratch: res, tx and conv scratch are used one at a time
  size_t shared = max_res;
  if (max_tx > shared) shared = max_tx;
  if (max_conv > shared) shared = max_conv;
  uint8_t* sh = static_cast<uint8_t*>(ar.take(shared + 4096));
  p->conv_scratch = reinterpret_cast<bf16*>(sh);
  (void)sh;
  return ar.off;
}

struct VaePlan {
  Ctx c;
  bf16 *pp[2];
  bf16* shared;  // resblock / attention / resampling / conv_in scratch, used one at a time
  size_t shared_bytes;
};

size_t plan_vae(Arena& ar, const sd_vae_cfg* cfg, cudaStream_t st, int sms, VaePlan* p) {
  const int L = cfg->n_levels;
  std::vector<int> ch;
  for (int l = L - 1; l >= 0; --l) ch.push_back(cfg->block_channels[l]);
  p->c = make_ctx(ar, st, sms);
  auto rnd = [](size_t b) { return (b + 255) / 256 * 256; };
  size_t H = cfg->height, Wd = cfg->width;
  size_t max_act = H * Wd * ch[0];
  size_t need = rnd(H * Wd * cfg->latent_channels * 2) + rnd(H * Wd * conv_in_kp(cfg->latent_channels) * 2);
  {
    Arena a{nullptr, 0};
    plan_vae_attn_scratch(a, (int64_t)(H * Wd), ch[0]);
    need = std::max(need, a.off + 1024);
  }
  int c_prev = ch[0];
  auto res_need = [&](size_t hw, int ci, int co) {
    need = std::max(need, rnd(hw * ci * 2) + 2 * rnd(hw * co * 2) + 1024);
    max_act = std::max(max_act, hw * (size_t)co);
  };
  res_need(H * Wd, c_prev, c_prev);
  for (int i = 0; i < L; ++i) {
    for (int j = 0; j <= cfg->layers_per_block; ++j) {
      res_need(H * Wd, c_prev, ch[i]);
      c_prev = ch[i];
    }
    if (i < L - 1) {
      need = std::max(need, rnd(4 * H * Wd * ch[i] * 2) + 1024);  // materialised nearest-2x input
      H *= 2;
      Wd *= 2;
      max_act = std::max(max_act, H * Wd * (size_t)ch[i]);
    }
  }
  need = std::max(need, rnd(H * Wd * ch[L - 1] * 2) + 1024);  // output head GroupNorm
  p->pp[0] = ar.bf(max_act);
  p->pp[1] = ar.bf(max_act);
  p->shared = static_cast<bf16*>(ar.take(need));
  p->shared_bytes = need;
  return ar.off;
}

// Carve module scratch out of the shared region at run time.
ResScratch carve_res(uint8_t* base, int hw, int cin, int cout) {
  Arena a{base, 0};
  return plan_res_scratch(a, hw, cin, cout);
}
TxScratch carve_tx(uint8_t* base, int hw, int C, int ctx_len) {
  Arena a{base, 0};
  return plan_tx_scratch(a, hw, C, ctx_len);
}

sd_status check_ws(size_t need, const void* ws, size_t ws_bytes) {
  if (!ws) return SD_ERR_NULL_ARG;
  if (!aligned16(ws)) return SD_ERR_MISALIGNED;
  if (ws_bytes < need) return SD_ERR_WORKSPACE_TOO_SMALL;
  return SD_OK;
}

// Zero the device error word and this call's GroupNorm accumulators.
sd_status clear_header(const Ctx& c) {
  if (cudaMemsetAsync(c.err, 0, c.clear_bytes, c.st) != cudaSuccess) return SD_ERR_LAUNCH;
  return SD_OK;
}

}  // namespace

// ====================================================================== exported
extern "C" {

const char* sd_version(void) { return "sd-b200 0.1"; }

sd_status sd_gemm_override(int32_t bn, int32_t splits) {
  const bool bn_ok = bn == 0 || (bn >= 32 && bn <= 256 && bn % 32 == 0);
  if (!bn_ok || splits < 0 || splits > 16) return SD_ERR_UNSUPPORTED;
  g_force_bn.store(bn, std::memory_order_relaxed);
  g_force_splits.store(splits, std::memory_order_relaxed);
  return SD_OK;
}

const char* sd_status_string(sd_status s) {
  switch (s) {
    case SD_OK: return "ok";
    case SD_ERR_NULL_ARG: return "a required pointer is NULL";
    case SD_ERR_BAD_SHAPE: return "inconsistent shape";
    case SD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SD_ERR_MISALIGNED: return "device pointer not 16-byte aligned";
    case SD_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case SD_ERR_NOT_SM100: return "device is not compute capability 10.0 (B200)";
    case SD_ERR_LAUNCH: return "kernel launch or CUDA runtime call failed";
    case SD_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case SD_ERR_CAPACITY: return "output table too small";
  }
  return "unknown status";
}

// ------------------------------------------------------------------ layouts / packing
sd_status sd_time_weight_layout(const sd_time_cfg* cfg, sd_tensor_desc* out, int32_t capacity, int32_t* n,
                                int64_t* ce, int64_t* pb) {
  sd_status s = check_time(cfg);
  if (s != SD_OK) return s;
  Table t;
  add_time(t, "time", cfg->proj_dim, cfg->temb_dim);
  return export_table(t, out, capacity, n, ce, pb);
}

static void conv_table(Table& t, const sd_conv_cfg* cfg, int kind) {
  switch (kind) {
    case SD_CONV_IN: add_conv_in(t, "conv_in", cfg->c_in, cfg->c_out, conv_in_kp(cfg->c_in)); break;
    case SD_CONV_DOWNSAMPLE: add_conv3x3(t, "down", cfg->c_in, cfg->c_out); break;
    case SD_CONV_UPSAMPLE: add_conv3x3(t, "up", cfg->c_in, cfg->c_out); break;
    default: add_output(t, cfg->c_in, cfg->c_out); break;
  }
}

sd_status sd_conv_weight_layout(const sd_conv_cfg* cfg, int32_t kind, sd_tensor_desc* out, int32_t capacity,
                                int32_t* n, int64_t* ce, int64_t* pb) {
  sd_status s = check_conv(cfg, kind);
  if (s != SD_OK) return s;
  Table t;
  conv_table(t, cfg, kind);
  return export_table(t, out, capacity, n, ce, pb);
}

sd_status sd_resblock_weight_layout(const sd_resblock_cfg* cfg, sd_tensor_desc* out, int32_t capacity, int32_t* n,
                                    int64_t* ce, int64_t* pb) {
  sd_status s = check_res(cfg);
  if (s != SD_OK) return s;
  Table t;
  add_resblock(t, "res", cfg->c_x + cfg->c_skip, cfg->c_out, cfg->temb_dim);
  return export_table(t, out, capacity, n, ce, pb);
}

sd_status sd_transformer_weight_layout(const sd_transformer_cfg* cfg, sd_tensor_desc* out, int32_t capacity,
                                       int32_t* n, int64_t* ce, int64_t* pb) {
  sd_status s = check_tx(cfg);
  if (s != SD_OK) return s;
  Table t;
  add_transformer(t, "attn", cfg->channels, cfg->depth, cfg->ctx_dim);
  return export_table(t, out, capacity, n, ce, pb);
}

sd_status sd_unet_weight_layout(const sd_unet_cfg* cfg, sd_tensor_desc* out, int32_t capacity, int32_t* n,
                                int64_t* ce, int64_t* pb) {
  sd_status s = check_unet(cfg);
  if (s != SD_OK) return s;
  Table t;
  add_unet(t, *cfg);
  return export_table(t, out, capacity, n, ce, pb);
}

sd_status sd_time_pack_weights(const sd_time_cfg* cfg, const uint16_t* canon, void* packed) {
  sd_status s = check_time(cfg);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  add_time(t, "time", cfg->proj_dim, cfg->temb_dim);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

sd_status sd_conv_pack_weights(const sd_conv_cfg* cfg, int32_t kind, const uint16_t* canon, void* packed) {
  sd_status s = check_conv(cfg, kind);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  conv_table(t, cfg, kind);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

sd_status sd_resblock_pack_weights(const sd_resblock_cfg* cfg, const uint16_t* canon, void* packed) {
  sd_status s = check_res(cfg);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  add_resblock(t, "res", cfg->c_x + cfg->c_skip, cfg->c_out, cfg->temb_dim);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

sd_status sd_transformer_pack_weights(const sd_transformer_cfg* cfg, const uint16_t* canon, void* packed) {
  sd_status s = check_tx(cfg);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  add_transformer(t, "attn", cfg->channels, cfg->depth, cfg->ctx_dim);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

sd_status sd_unet_pack_weights(const sd_unet_cfg* cfg, const uint16_t* canon, void* packed) {
  sd_status s = check_unet(cfg);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  add_unet(t, *cfg);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

// ------------------------------------------------------------------ workspace sizes
size_t sd_time_workspace_size(const sd_time_cfg* cfg) {
  if (check_time(cfg) != SD_OK) return 0;
  Arena a{nullptr, 0};
  TimePlan p;
  return plan_time(a, cfg, nullptr, kMaxStatBlocks, &p);
}
size_t sd_conv_workspace_size(const sd_conv_cfg* cfg, int32_t kind) {
  if (check_conv(cfg, kind) != SD_OK) return 0;
  Arena a{nullptr, 0};
  ConvPlan p;
  return plan_conv(a, cfg, kind, nullptr, kMaxStatBlocks, &p);
}
size_t sd_resblock_workspace_size(const sd_resblock_cfg* cfg) {
  if (check_res(cfg) != SD_OK) return 0;
  Arena a{nullptr, 0};
  ResPlan p;
  return plan_res(a, cfg, nullptr, kMaxStatBlocks, &p);
}
size_t sd_transformer_workspace_size(const sd_transformer_cfg* cfg) {
  if (check_tx(cfg) != SD_OK) return 0;
  Arena a{nullptr, 0};
  TxPlan p;
  return plan_tx(a, cfg, nullptr, kMaxStatBlocks, &p);
}
size_t sd_unet_workspace_size(const sd_unet_cfg* cfg) {
  if (check_unet(cfg) != SD_OK) return 0;
  Arena a{nullptr, 0};
  UNetPlan p;
  return plan_unet(a, cfg, nullptr, kMaxStatBlocks, &p);
}

// ------------------------------------------------------------------ forward calls
sd_status sd_time_embed(const sd_time_cfg* cfg, const void* pw, float timestep, float* temb, void* ws,
                        size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_time(cfg);
  if (s != SD_OK) return s;
  if (!pw || !temb) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(temb)) return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_time_workspace_size(cfg), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  TimePlan p;
  plan_time(a, cfg, (cudaStream_t)stream, d.sms, &p);
  if ((s = clear_header(p.c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  int rs_clean = 0;  // both row-statistics buffers are zeroed with the header
  p.c.rs_clean = &rs_clean;
  Table tab;
  TimeW w = add_time(tab, "time", cfg->proj_dim, cfg->temb_dim);
  return run_time(p.c, w, pw, cfg->proj_dim, cfg->temb_dim, timestep, p.phi, p.hid, temb);
}

sd_status sd_conv_fwd(const sd_conv_cfg* cfg, int32_t kind, const void* pw, const void* x0, const void* x1,
                      const void* x2, void* y, void* ws, size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_conv(cfg, kind);
  if (s != SD_OK) return s;
  if (!pw || !x0 || !y) return SD_ERR_NULL_ARG;
  const bool three = (kind == SD_CONV_IN && cfg->c_in == 9);
  if (three && (!x1 || !x2)) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(x0) || !aligned16(y) || (three && (!aligned16(x1) || !aligned16(x2))))
    return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_conv_workspace_size(cfg, kind), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  ConvPlan p;
  plan_conv(a, cfg, kind, (cudaStream_t)stream, d.sms, &p);
  if ((s = clear_header(p.c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  int rs_clean = 0;  // both row-statistics buffers are zeroed with the header
  p.c.rs_clean = &rs_clean;
  Table tab;
  const int H = cfg->height, Wd = cfg->width;
  const bf16* X0 = static_cast<const bf16*>(x0);
  bf16* Y = static_cast<bf16*>(y);
  switch (kind) {
    case SD_CONV_IN: {
      ConvW w = add_conv_in(tab, "conv_in", cfg->c_in, cfg->c_out, conv_in_kp(cfg->c_in));
      if (three)
        return run_conv_in(p.c, w, pw, conv_in_kp(9), H, Wd, X0, 4, static_cast<const bf16*>(x1), 4,
                           static_cast<const bf16*>(x2), 1, cfg->c_out, Y, p.scratch);
      return run_conv_in(p.c, w, pw, conv_in_kp(cfg->c_in), H, Wd, X0, cfg->c_in, nullptr, 0, nullptr, 0,
                         cfg->c_out, Y, p.scratch);
    }
    case SD_CONV_DOWNSAMPLE: {
      ConvW w = add_conv3x3(tab, "down", cfg->c_in, cfg->c_out);
      return run_downsample(p.c, w, pw, H, Wd, cfg->c_in, X0, Y, p.scratch);
    }
    case SD_CONV_UPSAMPLE: {
      ConvW w = add_conv3x3(tab, "up", cfg->c_in, cfg->c_out);
      return run_upsample(p.c, w, pw, H, Wd, cfg->c_in, X0, Y, p.scratch);
    }
    default: {
      OutW w = add_output(tab, cfg->c_in, cfg->c_out);
      return run_output(p.c, w, pw, H, Wd, cfg->c_in, cfg->c_out, cfg->groups, cfg->eps, X0, Y, p.scratch);
    }
  }
}

sd_status sd_resblock_fwd(const sd_resblock_cfg* cfg, const void* pw, const void* x, const void* skip,
                          const float* temb, void* y, void* ws, size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_res(cfg);
  if (s != SD_OK) return s;
  if (!pw || !x || !temb || !y || (cfg->c_skip > 0 && !skip)) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(x) || !aligned16(y) || !aligned16(temb) || (skip && !aligned16(skip)))
    return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_resblock_workspace_size(cfg), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  ResPlan p;
  plan_res(a, cfg, (cudaStream_t)stream, d.sms, &p);
  if ((s = clear_header(p.c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  int rs_clean = 0;  // both row-statistics buffers are zeroed with the header
  p.c.rs_clean = &rs_clean;
  Table tab;
  ResW w = add_resblock(tab, "res", cfg->c_x + cfg->c_skip, cfg->c_out, cfg->temb_dim);
  sdk::GemvBatch b;
  memset(&b, 0, sizeof(b));
  b.njobs = 1;
  b.K = cfg->temb_dim;
  b.silu_in = 1;
  b.x = temb;
  b.job[0] = {W(pw, w.tw), W(pw, w.tb), p.tproj, cfg->c_out};
  CK(run_gemv(p.c, b));
  return run_resblock(p.c, w, pw, cfg->height, cfg->width, static_cast<const bf16*>(x), cfg->c_x,
                      static_cast<const bf16*>(skip), cfg->c_skip, p.tproj, cfg->groups, cfg->eps,
                      static_cast<bf16*>(y), p.s);
}

sd_status sd_transformer_fwd(const sd_transformer_cfg* cfg, const void* pw, const void* x, const void* context,
                             void* y, void* ws, size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_tx(cfg);
  if (s != SD_OK) return s;
  if (!pw || !x || !context || !y) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(x) || !aligned16(y) || !aligned16(context)) return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_transformer_workspace_size(cfg), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  TxPlan p;
  plan_tx(a, cfg, (cudaStream_t)stream, d.sms, &p);
  if ((s = clear_header(p.c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  int rs_clean = 0;  // both row-statistics buffers are zeroed with the header
  p.c.rs_clean = &rs_clean;
  Table tab;
  TxW w = add_transformer(tab, "attn", cfg->channels, cfg->depth, cfg->ctx_dim);
  return run_transformer(p.c, w, pw, cfg->height, cfg->width, static_cast<const bf16*>(x),
                         static_cast<const bf16*>(context), cfg->ctx_len, cfg->groups, cfg->gn_eps, cfg->ln_eps,
                         static_cast<bf16*>(y), p.s);
}

sd_status sd_unet_step(const sd_unet_cfg* cfg, const void* pw, const void* latent, float timestep,
                       const void* context, void* eps_out, void* ws, size_t ws_bytes, sd_stream_t stream) {
  return sd_unet_step_cond(cfg, pw, latent, timestep, context, nullptr, nullptr, eps_out, ws, ws_bytes, stream);
}

sd_status sd_unet_step_cond(const sd_unet_cfg* cfg, const void* pw, const void* latent, float timestep,
                            const void* context, const void* add_text, const float* add_time_ids, void* eps_out,
                            void* ws, size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_unet(cfg);
  if (s != SD_OK) return s;
  if (!pw || !latent || !context || !eps_out) return SD_ERR_NULL_ARG;
  if (cfg->add_text_dim > 0 && (!add_text || (cfg->add_time_ids > 0 && !add_time_ids))) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(latent) || !aligned16(context) || !aligned16(eps_out) ||
      (add_text && cfg->add_text_dim > 0 && !aligned16(add_text)))
    return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_unet_workspace_size(cfg), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  UNetPlan p;
  plan_unet(a, cfg, (cudaStream_t)stream, d.sms, &p);
  const Ctx& c = p.c;
  if ((s = clear_header(c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  int rs_clean = 0;  // both row-statistics buffers are zeroed with the header
  p.c.rs_clean = &rs_clean;
  Table tab;
  UNetW u = add_unet(tab, *cfg);
  const int L = cfg->n_levels;
  const int* ch = cfg->block_channels;
  const int G = cfg->groups;
  const float eps = cfg->eps;
  const bf16* ctx = static_cast<const bf16*>(context);
  uint8_t* shared = reinterpret_cast<uint8_t*>(p.conv_scratch);

  // the context K/V of every cross-attention in one GEMM (the context is the same for all of them)
  if (u.ctx_kv_w < 0 || u.ctx_k_cols != p.ctx_k_cols) return SD_ERR_UNSUPPORTED;
  if ((s = run_linear(c, ctx, cfg->ctx_len, cfg->ctx_dim, W(pw, u.ctx_kv_w), 2 * p.ctx_k_cols, nullptr, nullptr, 0,
                      p.ctx_kv, 2 * p.ctx_k_cols, sdk::GEMM_PLAIN, 0, nullptr, p.ctx_k_cols)) != SD_OK)  // V as FP16
    return s;
  const CtxKV pre{p.ctx_kv, 2 * p.ctx_k_cols, p.ctx_k_cols};
  // time embedding and every resblock's projection of SiLU(temb), batched
  if ((s = run_time(c, u.time, pw, cfg->time_proj_dim, cfg->temb_dim, timestep, p.phi, p.hid, p.temb)) != SD_OK)
    return s;
  if (u.has_add) {
    // temb += Linear(SiLU(Linear([text | phi(id_0) | ...])))
    sdk::AddIds ids;
    memset(&ids, 0, sizeof(ids));
    for (int i = 0; i < cfg->add_time_ids; ++i) ids.v[i] = add_time_ids[i];
    const int dim = cfg->add_text_dim + cfg->add_time_ids * cfg->add_time_dim;
    {
      sdp::Scope sc("add_embed_input", sdp::F_OTHER, 0, 2.0 * cfg->add_text_dim + 4.0 * dim, c.st);
      CK(sdk::launch_add_embed_input(static_cast<const bf16*>(add_text), cfg->add_text_dim, ids, cfg->add_time_ids,
                                     cfg->add_time_dim, p.add_x, c.st));
    }
    sdk::GemvBatch b;
    memset(&b, 0, sizeof(b));
    b.njobs = 1;
    b.K = dim;
    b.silu_out = 1;
    b.x = p.add_x;
    b.job[0] = {W(pw, u.add.l1w), W(pw, u.add.l1b), p.add_h, cfg->temb_dim};
    CK(run_gemv(c, b));
    b.K = cfg->temb_dim;
    b.silu_out = 0;
    b.accum_out = 1;
    b.x = p.add_h;
    b.job[0] = {W(pw, u.add.l2w), W(pw, u.add.l2b), p.temb, cfg->temb_dim};
    CK(run_gemv(c, b));
  }
  std::vector<const ResW*> all_res;
  for (auto& lv : u.down)
    for (auto& r : lv.res) all_res.push_back(&r);
  all_res.push_back(&u.mid_res0);
  all_res.push_back(&u.mid_res1);
  for (auto& lv : u.up)
    for (auto& r : lv.res) all_res.push_back(&r);
  std::vector<float*> tproj(all_res.size());
  {
    float* tp = p.tproj;
    for (size_t i = 0; i < all_res.size(); ++i) {
      tproj[i] = tp;
      tp += all_res[i]->c_out;
    }
    for (size_t i0 = 0; i0 < all_res.size(); i0 += sdk::kMaxGemvJobs) {
      sdk::GemvBatch b;
      memset(&b, 0, sizeof(b));
      b.K = cfg->temb_dim;
      b.silu_in = 1;
      b.x = p.temb;
      for (size_t i = i0; i < all_res.size() && b.njobs < sdk::kMaxGemvJobs; ++i)
        b.job[b.njobs++] = {W(pw, all_res[i]->tw), W(pw, all_res[i]->tb), tproj[i], all_res[i]->c_out};
      CK(run_gemv(c, b));
    }
  }
  size_t ri = 0;
  int H = cfg->height, Wd = cfg->width;
  // conv_in -> skip 0
  if ((s = run_conv_in(c, u.conv_in, pw, u.conv_in_kp, H, Wd, static_cast<const bf16*>(latent), cfg->in_channels,
                       nullptr, 0, nullptr, 0, ch[0], p.skip[0], reinterpret_cast<bf16*>(shared))) != SD_OK)
    return s;
  size_t si = 1;
  const bf16* h = p.skip[0];
  int hc = ch[0];
  for (int l = 0; l < L; ++l) {
    const auto& lv = u.down[l];
    for (int i = 0; i < cfg->layers_per_block; ++i) {
      bf16* dst = p.skip[si++];
      ResScratch rs = carve_res(shared, H * Wd, hc, ch[l]);
      if ((s = run_resblock(c, lv.res[i], pw, H, Wd, h, hc, nullptr, 0, tproj[ri++], G, eps, dst, rs)) != SD_OK)
        return s;
      if (!lv.attn.empty()) {
        TxScratch ts = carve_tx(shared, H * Wd, ch[l], cfg->ctx_len);
        if ((s = run_transformer(c, lv.attn[i], pw, H, Wd, dst, ctx, cfg->ctx_len, G, eps, eps, dst, ts, &pre)) != SD_OK)
          return s;
      }
      h = dst;
      hc = ch[l];
    }
    if (lv.has_down) {
      bf16* dst = p.skip[si++];
      if ((s = run_downsample(c, lv.down, pw, H, Wd, hc, h, dst, reinterpret_cast<bf16*>(shared))) != SD_OK) return s;
      H /= 2;
      Wd /= 2;
      h = dst;
    }
  }
  // mid
  {
    ResScratch rs = carve_res(shared, H * Wd, hc, hc);
    if ((s = run_resblock(c, u.mid_res0, pw, H, Wd, h, hc, nullptr, 0, tproj[ri++], G, eps, p.mid_a, rs)) != SD_OK)
      return s;
    TxScratch ts = carve_tx(shared, H * Wd, hc, cfg->ctx_len);
    if ((s = run_transformer(c, u.mid_attn, pw, H, Wd, p.mid_a, ctx, cfg->ctx_len, G, eps, eps, p.mid_a, ts, &pre)) !=
        SD_OK)
      return s;
    if ((s = run_resblock(c, u.mid_res1, pw, H, Wd, p.mid_a, hc, nullptr, 0, tproj[ri++], G, eps, p.mid_b, rs)) !=
        SD_OK)
      return s;
    h = p.mid_b;
  }
  // up
  int pi = 0;
  for (int up = 0; up < L; ++up) {
    const int l = L - 1 - up;
    const auto& lv = u.up[up];
    for (int i = 0; i <= cfg->layers_per_block; ++i) {
      --si;
      const bf16* sk = p.skip[si];
      const int cs = p.skip_c[si];
      bf16* dst = p.pp[pi];
      pi ^= 1;
      ResScratch rs = carve_res(shared, H * Wd, hc + cs, ch[l]);
      if ((s = run_resblock(c, lv.res[i], pw, H, Wd, h, hc, sk, cs, tproj[ri++], G, eps, dst, rs)) != SD_OK) return s;
      if (!lv.attn.empty()) {
        TxScratch ts = carve_tx(shared, H * Wd, ch[l], cfg->ctx_len);
        if ((s = run_transformer(c, lv.attn[i], pw, H, Wd, dst, ctx, cfg->ctx_len, G, eps, eps, dst, ts, &pre)) != SD_OK)
          return s;
      }
      h = dst;
      hc = ch[l];
    }
    if (lv.has_up) {
      bf16* dst = p.pp[pi];
      pi ^= 1;
      if ((s = run_upsample(c, lv.up, pw, H, Wd, hc, h, dst, reinterpret_cast<bf16*>(shared))) != SD_OK) return s;
      H *= 2;
      Wd *= 2;
      h = dst;
    }
  }
  return run_output(c, u.out, pw, H, Wd, hc, cfg->out_channels, G, eps, h, static_cast<bf16*>(eps_out),
                    reinterpret_cast<bf16*>(shared));
}

sd_status sd_vae_weight_layout(const sd_vae_cfg* cfg, sd_tensor_desc* out, int32_t capacity, int32_t* n, int64_t* ce,
                               int64_t* pb) {
  sd_status s = check_vae(cfg);
  if (s != SD_OK) return s;
  Table t;
  add_vae(t, *cfg);
  return export_table(t, out, capacity, n, ce, pb);
}

sd_status sd_vae_pack_weights(const sd_vae_cfg* cfg, const uint16_t* canon, void* packed) {
  sd_status s = check_vae(cfg);
  if (s != SD_OK) return s;
  if (!canon || !packed) return SD_ERR_NULL_ARG;
  Table t;
  add_vae(t, *cfg);
  pack(t, canon, static_cast<uint8_t*>(packed));
  return SD_OK;
}

size_t sd_vae_workspace_size(const sd_vae_cfg* cfg) {
  if (check_vae(cfg) != SD_OK) return 0;
  Arena a{nullptr, 0};
  VaePlan p;
  return plan_vae(a, cfg, nullptr, kMaxStatBlocks, &p);
}

sd_status sd_vae_decode(const sd_vae_cfg* cfg, const void* pw, const void* latent, void* image, void* ws,
                        size_t ws_bytes, sd_stream_t stream) {
  sd_status s = check_vae(cfg);
  if (s != SD_OK) return s;
  if (!pw || !latent || !image) return SD_ERR_NULL_ARG;
  if (!aligned16(pw) || !aligned16(latent) || !aligned16(image)) return SD_ERR_MISALIGNED;
  if ((s = check_ws(sd_vae_workspace_size(cfg), ws, ws_bytes)) != SD_OK) return s;
  DevInfo d;
  if ((s = device_info(&d)) != SD_OK) return s;
  Arena a{static_cast<uint8_t*>(ws), 0};
  VaePlan p;
  plan_vae(a, cfg, (cudaStream_t)stream, d.sms, &p);
  const Ctx& c = p.c;
  if ((s = clear_header(c)) != SD_OK) return s;
  int gn_seq = 0;
  p.c.gn_seq = &gn_seq;
  Table tab;
  const VaeW v = add_vae(tab, *cfg);
  const int G = cfg->groups, L = cfg->n_levels;
  const float eps = cfg->eps;
  int H = cfg->height, Wd = cfg->width;
  uint8_t* sh = reinterpret_cast<uint8_t*>(p.shared);
  // latent / scaling factor -> 1x1 post-quantisation conv -> conv_in
  {
    const int lc = cfg->latent_channels;
    bf16* lat = reinterpret_cast<bf16*>(sh);
    bf16* col = reinterpret_cast<bf16*>(sh + ((size_t)H * Wd * lc * 2 + 255) / 256 * 256);
    {
      sdp::Scope sc("vae_latent_in", sdp::F_OTHER, 0, 4.0 * H * Wd * lc, c.st);
      CK(sdk::launch_vae_latent_in(static_cast<const bf16*>(latent), W(pw, v.post_quant.w), W(pw, v.post_quant.b), lc,
                                   (int64_t)H * Wd, 1.0f / cfg->scaling_factor, lat, c.st));
    }
    if ((s = run_conv_in(c, v.conv_in, pw, v.conv_in_kp, H, Wd, lat, lc, nullptr, 0, nullptr, 0,
                         v.up[0].C, p.pp[0], col)) != SD_OK)
      return s;
  }
  int cur = 0;
  auto res = [&](const ResW& w, int cx) -> sd_status {
    ResScratch rs = carve_res(sh, H * Wd, cx, w.c_out);
    sd_status r = run_resblock(c, w, pw, H, Wd, p.pp[cur], cx, nullptr, 0, nullptr, G, eps, p.pp[cur ^ 1], rs);
    cur ^= 1;
    return r;
  };
  int C = v.up[0].C;
  if ((s = res(v.mid_res0, C)) != SD_OK) return s;
  {
    Arena aa{sh, 0};
    const VaeAttnScratch as = plan_vae_attn_scratch(aa, (int64_t)H * Wd, C);
    if ((s = run_vae_attention(c, v.mid_attn, pw, H, Wd, G, eps, p.pp[cur], p.pp[cur ^ 1], as)) != SD_OK) return s;
    cur ^= 1;
  }
  if ((s = res(v.mid_res1, C)) != SD_OK) return s;
  for (int i = 0; i < L; ++i) {
    for (const ResW& w : v.up[i].res) {
      if ((s = res(w, C)) != SD_OK) return s;
      C = w.c_out;
    }
    if (v.up[i].has_up) {
      if ((s = run_upsample(c, v.up[i].up, pw, H, Wd, C, p.pp[cur], p.pp[cur ^ 1], reinterpret_cast<bf16*>(sh))) !=
          SD_OK)
        return s;
      cur ^= 1;
      H *= 2;
      Wd *= 2;
    }
  }
  return run_output(c, v.out, pw, H, Wd, C, cfg->out_channels, G, eps, p.pp[cur], static_cast<bf16*>(image),
                    reinterpret_cast<bf16*>(sh));
}

sd_status sd_record_begin(void* dev_buf, size_t bytes) {
  if (!dev_buf && bytes) return SD_ERR_NULL_ARG;
  if (!aligned16(dev_buf)) return SD_ERR_MISALIGNED;
  Recorder& r = t_rec;
  r.on = true;
  r.buf = static_cast<uint8_t*>(dev_buf);
  r.bytes = bytes;
  r.used = 0;
  r.overflow = false;
  r.res_count = r.tx_count = 0;
  r.entries.clear();
  return SD_OK;
}

sd_status sd_record_end(int32_t* n_entries) {
  Recorder& r = t_rec;
  r.on = false;
  if (n_entries) *n_entries = (int32_t)r.entries.size();
  return r.overflow ? SD_ERR_CAPACITY : SD_OK;
}

sd_status sd_record_read(sd_record_entry* out, int32_t capacity, int32_t* n) {
  const Recorder& r = t_rec;
  if (n) *n = (int32_t)r.entries.size();
  if (!out) return SD_OK;
  if (capacity < (int32_t)r.entries.size()) return SD_ERR_CAPACITY;
  for (size_t i = 0; i < r.entries.size(); ++i) out[i] = r.entries[i];
  return SD_OK;
}

sd_status sd_debug_inject_timeout(int32_t n_launches, int32_t spin_limit) {
  if (n_launches < 0 || (n_launches > 0 && (spin_limit < 1 || spin_limit > (1 << 24)))) return SD_ERR_UNSUPPORTED;
  g_inject_spins.store(spin_limit, std::memory_order_relaxed);
  g_inject_n.store(n_launches, std::memory_order_relaxed);
  return SD_OK;
}

sd_status sd_query_device_status(void* ws, sd_stream_t stream) {
  if (!ws) return SD_ERR_NULL_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SD_ERR_LAUNCH;
  int word = 0;
  if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SD_ERR_LAUNCH;
  if (word != 0) {
    cudaMemset(ws, 0, sizeof(int));
    return SD_ERR_DEVICE_TIMEOUT;
  }
  return SD_OK;
}

}  // extern "C"
