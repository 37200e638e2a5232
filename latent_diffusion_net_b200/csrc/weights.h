// Weight tables: the canonical tensor list of every module (names, shapes,
// kinds, fan-in) and the packed layout the kernels read. Pure host code.
#pragma once

#include <stdint.h>

#include <string>
#include <vector>

#include "sd_api.h"

namespace sdw {

enum Pack : int {
  PACK_COPY = 0,     // same element order
  PACK_CONV_KRSC,    // [O][C][kh][kw] -> [O][kh][kw][C]
  PACK_CONV_IM2COL,  // [O][C][3][3]  -> [O][Kp], k = (ky*3+kx)*C + c, zero-padded to Kp
  PACK_GEGLU_ROWS,   // [8C][C]: row 2j = value row j, row 2j+1 = gate row 4C + j
  PACK_GEGLU_BIAS,   // [8C]: same interleave
  PACK_LNFOLD,       // [R][K] times the LayerNorm gamma of tensor `aux` along K, rounded to BF16
  PACK_LNFOLD_GEGLU  // PACK_GEGLU_ROWS of the PACK_LNFOLD product
};

// FP32 vectors derived from several canonical tensors (packed after them): for
// a linear layer fed by a LayerNorm, with W' = W * gamma (as packed),
// c1[r] = sum_k W'[r][k] and c2[r] = sum_k W[r][k] * beta[k] + bias[r].
struct Derived {
  bool c2;          // false: c1 from the packed W'; true: c2 from canonical W, beta, bias
  int64_t out_off;  // packed byte offset of the FP32 vector
  int64_t rows, K;
  int w_tensor;     // first canonical tensor of the rows (consecutive tensors continue them)
  int beta_tensor;  // c2: LayerNorm beta
  int bias_tensor;  // c2: bias or -1
  bool geglu;       // rows interleaved as PACK_GEGLU_ROWS
};

struct Tensor {
  std::string name;
  int ndim = 0;
  int64_t shape[4] = {0, 0, 0, 0};
  int kind = 0;
  int fan_in = 0;
  int64_t canon_off = 0;   // elements
  int64_t packed_off = 0;  // bytes
  int pack = PACK_COPY;
  int64_t packed_elems = 0;
  int aux = 0;  // PACK_CONV_IM2COL: Kp
  int64_t numel() const {
    int64_t n = 1;
    for (int i = 0; i < ndim; ++i) n *= shape[i];
    return n;
  }
};

struct Table {
  std::vector<Tensor> t;
  std::vector<Derived> d;
  int64_t canon_elems = 0;
  int64_t packed_bytes = 0;
  // Appends a tensor; returns its packed byte offset.
  int64_t add(const std::string& name, std::initializer_list<int64_t> shape, int kind, int fan_in,
              int pack = PACK_COPY, int aux = 0);
  // Appends a derived FP32 vector of `rows` entries; returns its packed byte offset.
  int64_t add_derived(const Derived& x);
  // Appends a tensor whose packed place is given later by place_run (canonical
  // order is unchanged); returns its index.
  int add_deferred(const std::string& name, std::initializer_list<int64_t> shape, int kind, int fan_in);
  // Places the deferred tensors `idx` back to back (one matrix when they share
  // their row length and each is a multiple of 256 bytes); returns the offset of the first.
  int64_t place_run(const std::vector<int>& idx);
  int last() const { return (int)t.size() - 1; }
};

// Packed byte offsets of each module's tensors.
struct TimeW {
  int64_t l1w, l1b, l2w, l2b;
};
struct ConvW {
  int64_t w, b;
};
struct OutW {
  int64_t ng, nb, w, b;
};
struct ResW {
  int c_in, c_out;
  int64_t n1g, n1b, c1w, c1b, tw, tb, n2g, n2b, c2w, c2b, sw, sb;  // sw/sb = -1 without shortcut
};
struct TxBlockW {
  // kv2 = -1 when the cross-attention K/V weights live in the whole model's context
  // K/V matrix instead (ctx_k_col = this block's first K column there)
  int64_t ln1g, ln1b, qkv, o1w, o1b, ln2g, ln2b, q2, kv2, o2w, o2b, ln3g, ln3b, f1w, f1b, f2w, f2b;
  int ctx_k_col = -1;
  // LayerNorm folded into the following linear: qkv, q2 and f1w are packed as
  // W * gamma; c1 / c2 are the FP32 column terms of the GEMM epilogue
  int64_t qkv_c1, qkv_c2, q2_c1, q2_c2, f1_c1, f1_c2;
};
struct TxW {
  int C, depth, ctx_dim;
  int64_t ng, nb, piw, pib, pow_, pob;
  std::vector<TxBlockW> blocks;
};

TimeW add_time(Table& tab, const std::string& prefix, int proj_dim, int temb_dim);
ConvW add_conv3x3(Table& tab, const std::string& prefix, int c_in, int c_out);
ConvW add_conv_in(Table& tab, const std::string& prefix, int c_in, int c_out, int kp);
OutW add_output(Table& tab, int c_in, int c_out);
ResW add_resblock(Table& tab, const std::string& prefix, int c_in, int c_out, int temb_dim);
// The context K/V weights of every cross-attention of a model, gathered into one
// [K of all blocks | V of all blocks] x ctx_dim matrix so that one GEMM projects
// the context for all of them: `k`/`v` collect the deferred tensors, `cols` the K width.
struct CtxKVGather {
  std::vector<int> k, v;
  int cols = 0;
};
TxW add_transformer(Table& tab, const std::string& prefix, int C, int depth, int ctx_dim,
                    CtxKVGather* gather = nullptr);

// Whole U-Net: module order follows the forward pass.
struct UNetW {
  // context K/V of all cross-attentions: [2 * ctx_k_cols, ctx_dim] at ctx_kv_w (K rows first)
  int64_t ctx_kv_w = -1;
  int ctx_k_cols = 0;
  TimeW time;
  bool has_add;  // SDXL added conditioning MLP (same shape as the time MLP)
  TimeW add;
  ConvW conv_in;
  int conv_in_kp;
  struct Level {
    std::vector<ResW> res;
    std::vector<TxW> attn;  // empty when the level has no attention
    bool has_down;
    ConvW down;
  };
  std::vector<Level> down;
  ResW mid_res0, mid_res1;
  TxW mid_attn;
  struct UpLevel {
    std::vector<ResW> res;
    std::vector<TxW> attn;
    bool has_up;
    ConvW up;
  };
  std::vector<UpLevel> up;
  OutW out;
};
UNetW add_unet(Table& tab, const sd_unet_cfg& cfg);

// VAE decoder: resblocks without a time embedding (tw = tb = -1); the attention's
// q/k/v weights are one [3C, C] matrix and their biases one [3C] vector.
struct VaeAttnW {
  int C;
  int64_t ng, nb, qkv, qkv_b, ow, ob;
};
struct VaeW {
  ConvW post_quant;  // 1x1, [lc][lc]
  ConvW conv_in;
  int conv_in_kp;
  ResW mid_res0, mid_res1;
  VaeAttnW mid_attn;
  struct Level {
    std::vector<ResW> res;
    bool has_up;
    ConvW up;
    int C;
  };
  std::vector<Level> up;
  OutW out;
};
VaeW add_vae(Table& tab, const sd_vae_cfg& cfg);

int conv_in_kp(int c_in);

// Canonical (host, BF16 bits) -> packed (host).
void pack(const Table& tab, const uint16_t* canonical, uint8_t* packed);

sd_status export_table(const Table& tab, sd_tensor_desc* out, int32_t capacity, int32_t* n_tensors,
                       int64_t* canon_elems, int64_t* packed_bytes);

}  // namespace sdw
