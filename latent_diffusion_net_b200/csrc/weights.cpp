// Canonical parameter tables and packing. The canonical names, shapes and order
// are the interface shared with whoever fills the weights (the tests compare
// this table against an independent enumeration); the packed layout is private
// to the kernels.
#include "weights.h"

#include <string.h>

namespace sdw {

int64_t Table::add(const std::string& name, std::initializer_list<int64_t> shape, int kind, int fan_in, int pack,
                   int aux) {
  Tensor x;
  x.name = name;
  x.ndim = (int)shape.size();
  int i = 0;
  for (int64_t s : shape) x.shape[i++] = s;
  x.kind = kind;
  x.fan_in = fan_in;
  x.pack = pack;
  x.aux = aux;
  x.canon_off = canon_elems;
  canon_elems += x.numel();
  x.packed_elems = x.numel();
  if (pack == PACK_CONV_IM2COL) x.packed_elems = x.shape[0] * (int64_t)aux;
  packed_bytes = (packed_bytes + 255) & ~int64_t(255);
  x.packed_off = packed_bytes;
  packed_bytes += x.packed_elems * 2;
  t.push_back(x);
  return x.packed_off;
}

int Table::add_deferred(const std::string& name, std::initializer_list<int64_t> shape, int kind, int fan_in) {
  Tensor x;
  x.name = name;
  x.ndim = (int)shape.size();
  int i = 0;
  for (int64_t s : shape) x.shape[i++] = s;
  x.kind = kind;
  x.fan_in = fan_in;
  x.canon_off = canon_elems;
  canon_elems += x.numel();
  x.packed_elems = x.numel();
  x.packed_off = -1;
  t.push_back(x);
  return (int)t.size() - 1;
}

int64_t Table::place_run(const std::vector<int>& idx) {
  packed_bytes = (packed_bytes + 255) & ~int64_t(255);
  const int64_t first = packed_bytes;
  for (int i : idx) {
    t[i].packed_off = packed_bytes;
    packed_bytes += t[i].packed_elems * 2;
  }
  return first;
}

int64_t Table::add_derived(const Derived& x0) {
  Derived x = x0;
  packed_bytes = (packed_bytes + 255) & ~int64_t(255);
  x.out_off = packed_bytes;
  packed_bytes += x.rows * 4;
  d.push_back(x);
  return x.out_off;
}

TimeW add_time(Table& tab, const std::string& p, int proj, int temb) {
  TimeW w;
  w.l1w = tab.add(p + ".lin1.weight", {temb, proj}, SD_KIND_WEIGHT, proj);
  w.l1b = tab.add(p + ".lin1.bias", {temb}, SD_KIND_BIAS, proj);
  w.l2w = tab.add(p + ".lin2.weight", {temb, temb}, SD_KIND_WEIGHT, temb);
  w.l2b = tab.add(p + ".lin2.bias", {temb}, SD_KIND_BIAS, temb);
  return w;
}

ConvW add_conv3x3(Table& tab, const std::string& p, int ci, int co) {
  ConvW w;
  w.w = tab.add(p + ".weight", {co, ci, 3, 3}, SD_KIND_WEIGHT, ci * 9, PACK_CONV_KRSC);
  w.b = tab.add(p + ".bias", {co}, SD_KIND_BIAS, ci * 9);
  return w;
}

int conv_in_kp(int c_in) { return (9 * c_in + 63) / 64 * 64; }

ConvW add_conv_in(Table& tab, const std::string& p, int ci, int co, int kp) {
  ConvW w;
  w.w = tab.add(p + ".weight", {co, ci, 3, 3}, SD_KIND_WEIGHT, ci * 9, PACK_CONV_IM2COL, kp);
  w.b = tab.add(p + ".bias", {co}, SD_KIND_BIAS, ci * 9);
  return w;
}

OutW add_output(Table& tab, int ci, int co) {
  OutW w;
  w.ng = tab.add("out.norm.gamma", {ci}, SD_KIND_NORM_GAMMA, 0);
  w.nb = tab.add("out.norm.beta", {ci}, SD_KIND_NORM_BETA, 0);
  w.w = tab.add("conv_out.weight", {co, ci, 3, 3}, SD_KIND_WEIGHT, ci * 9, PACK_CONV_KRSC);
  w.b = tab.add("conv_out.bias", {co}, SD_KIND_BIAS, ci * 9);
  return w;
}

ResW add_resblock(Table& tab, const std::string& p, int ci, int co, int temb) {
  ResW w;
  w.c_in = ci;
  w.c_out = co;
  w.n1g = tab.add(p + ".norm1.gamma", {ci}, SD_KIND_NORM_GAMMA, 0);
  w.n1b = tab.add(p + ".norm1.beta", {ci}, SD_KIND_NORM_BETA, 0);
  w.c1w = tab.add(p + ".conv1.weight", {co, ci, 3, 3}, SD_KIND_WEIGHT, ci * 9, PACK_CONV_KRSC);
  w.c1b = tab.add(p + ".conv1.bias", {co}, SD_KIND_BIAS, ci * 9);
  w.tw = tab.add(p + ".temb.weight", {co, temb}, SD_KIND_WEIGHT, temb);
  w.tb = tab.add(p + ".temb.bias", {co}, SD_KIND_BIAS, temb);
  w.n2g = tab.add(p + ".norm2.gamma", {co}, SD_KIND_NORM_GAMMA, 0);
  w.n2b = tab.add(p + ".norm2.beta", {co}, SD_KIND_NORM_BETA, 0);
  w.c2w = tab.add(p + ".conv2.weight", {co, co, 3, 3}, SD_KIND_WEIGHT, co * 9, PACK_CONV_KRSC);
  w.c2b = tab.add(p + ".conv2.bias", {co}, SD_KIND_BIAS, co * 9);
  w.sw = w.sb = -1;
  if (ci != co) {
    w.sw = tab.add(p + ".skip.weight", {co, ci, 1, 1}, SD_KIND_WEIGHT, ci);
    w.sb = tab.add(p + ".skip.bias", {co}, SD_KIND_BIAS, ci);
  }
  return w;
}

TxW add_transformer(Table& tab, const std::string& p, int C, int depth, int D, CtxKVGather* gather) {
  TxW w;
  w.C = C;
  w.depth = depth;
  w.ctx_dim = D;
  w.ng = tab.add(p + ".norm.gamma", {C}, SD_KIND_NORM_GAMMA, 0);
  w.nb = tab.add(p + ".norm.beta", {C}, SD_KIND_NORM_BETA, 0);
  w.piw = tab.add(p + ".proj_in.weight", {C, C}, SD_KIND_WEIGHT, C);
  w.pib = tab.add(p + ".proj_in.bias", {C}, SD_KIND_BIAS, C);
  for (int d = 0; d < depth; ++d) {
    const std::string b = p + ".blocks." + std::to_string(d);
    TxBlockW k;
    k.ln1g = tab.add(b + ".ln1.gamma", {C}, SD_KIND_NORM_GAMMA, 0);
    const int ln1g = tab.last();
    k.ln1b = tab.add(b + ".ln1.beta", {C}, SD_KIND_NORM_BETA, 0);
    const int ln1b = tab.last();
    // q, k, v are consecutive (each a multiple of 256 bytes): one [3C, C] matrix, packed with LN1's gamma
    k.qkv = tab.add(b + ".attn1.q.weight", {C, C}, SD_KIND_WEIGHT, C, PACK_LNFOLD, ln1g);
    const int qkv = tab.last();
    tab.add(b + ".attn1.k.weight", {C, C}, SD_KIND_WEIGHT, C, PACK_LNFOLD, ln1g);
    tab.add(b + ".attn1.v.weight", {C, C}, SD_KIND_WEIGHT, C, PACK_LNFOLD, ln1g);
    k.o1w = tab.add(b + ".attn1.out.weight", {C, C}, SD_KIND_WEIGHT, C);
    k.o1b = tab.add(b + ".attn1.out.bias", {C}, SD_KIND_BIAS, C);
    k.ln2g = tab.add(b + ".ln2.gamma", {C}, SD_KIND_NORM_GAMMA, 0);
    const int ln2g = tab.last();
    k.ln2b = tab.add(b + ".ln2.beta", {C}, SD_KIND_NORM_BETA, 0);
    const int ln2b = tab.last();
    k.q2 = tab.add(b + ".attn2.q.weight", {C, C}, SD_KIND_WEIGHT, C, PACK_LNFOLD, ln2g);
    const int q2 = tab.last();
    if (gather) {
      // placed with every other block's K (and V) by the caller
      k.kv2 = -1;
      k.ctx_k_col = gather->cols;
      gather->cols += C;
      gather->k.push_back(tab.add_deferred(b + ".attn2.k.weight", {C, D}, SD_KIND_WEIGHT, D));
      gather->v.push_back(tab.add_deferred(b + ".attn2.v.weight", {C, D}, SD_KIND_WEIGHT, D));
    } else {
      // k, v of the cross-attention are consecutive: one [2C, D] matrix
      k.kv2 = tab.add(b + ".attn2.k.weight", {C, D}, SD_KIND_WEIGHT, D);
      tab.add(b + ".attn2.v.weight", {C, D}, SD_KIND_WEIGHT, D);
    }
    k.o2w = tab.add(b + ".attn2.out.weight", {C, C}, SD_KIND_WEIGHT, C);
    k.o2b = tab.add(b + ".attn2.out.bias", {C}, SD_KIND_BIAS, C);
    k.ln3g = tab.add(b + ".ln3.gamma", {C}, SD_KIND_NORM_GAMMA, 0);
    const int ln3g = tab.last();
    k.ln3b = tab.add(b + ".ln3.beta", {C}, SD_KIND_NORM_BETA, 0);
    const int ln3b = tab.last();
    k.f1w = tab.add(b + ".ff.w1.weight", {8 * C, C}, SD_KIND_WEIGHT, C, PACK_LNFOLD_GEGLU, ln3g);
    const int f1w = tab.last();
    k.f1b = tab.add(b + ".ff.w1.bias", {8 * C}, SD_KIND_BIAS, C, PACK_GEGLU_BIAS);
    const int f1b = tab.last();
    k.f2w = tab.add(b + ".ff.w2.weight", {C, 4 * C}, SD_KIND_WEIGHT, 4 * C);
    k.f2b = tab.add(b + ".ff.w2.bias", {C}, SD_KIND_BIAS, 4 * C);
    // column terms of the three folded LayerNorms, after the canonical tensors of this block
    k.qkv_c1 = tab.add_derived({false, 0, 3 * C, C, qkv, -1, -1, false});
    k.qkv_c2 = tab.add_derived({true, 0, 3 * C, C, qkv, ln1b, -1, false});
    k.q2_c1 = tab.add_derived({false, 0, C, C, q2, -1, -1, false});
    k.q2_c2 = tab.add_derived({true, 0, C, C, q2, ln2b, -1, false});
    k.f1_c1 = tab.add_derived({false, 0, 8 * C, C, f1w, -1, -1, true});
    k.f1_c2 = tab.add_derived({true, 0, 8 * C, C, f1w, ln3b, f1b, true});
    w.blocks.push_back(k);
  }
  w.pow_ = tab.add(p + ".proj_out.weight", {C, C}, SD_KIND_WEIGHT, C);
  w.pob = tab.add(p + ".proj_out.bias", {C}, SD_KIND_BIAS, C);
  return w;
}

UNetW add_unet(Table& tab, const sd_unet_cfg& cfg) {
  UNetW u;
  CtxKVGather gather;
  const int L = cfg.n_levels;
  const int* ch = cfg.block_channels;
  u.time = add_time(tab, "time", cfg.time_proj_dim, cfg.temb_dim);
  u.has_add = cfg.add_text_dim > 0;
  if (u.has_add) u.add = add_time(tab, "add", cfg.add_text_dim + cfg.add_time_ids * cfg.add_time_dim, cfg.temb_dim);
  u.conv_in_kp = conv_in_kp(cfg.in_channels);
  u.conv_in = add_conv_in(tab, "conv_in", cfg.in_channels, ch[0], u.conv_in_kp);
  std::vector<int> skips;
  skips.push_back(ch[0]);
  int c_prev = ch[0];
  for (int l = 0; l < L; ++l) {
    UNetW::Level lv;
    for (int i = 0; i < cfg.layers_per_block; ++i) {
      const std::string p = "down." + std::to_string(l);
      lv.res.push_back(add_resblock(tab, p + ".res." + std::to_string(i), c_prev, ch[l], cfg.temb_dim));
      c_prev = ch[l];
      if (cfg.attn_depth[l] > 0)
        lv.attn.push_back(
            add_transformer(tab, p + ".attn." + std::to_string(i), ch[l], cfg.attn_depth[l], cfg.ctx_dim, &gather));
      skips.push_back(ch[l]);
    }
    lv.has_down = l < L - 1;
    if (lv.has_down) {
      lv.down = add_conv3x3(tab, "down." + std::to_string(l) + ".down", ch[l], ch[l]);
      skips.push_back(ch[l]);
    }
    u.down.push_back(lv);
  }
  u.mid_res0 = add_resblock(tab, "mid.res.0", ch[L - 1], ch[L - 1], cfg.temb_dim);
  u.mid_attn = add_transformer(tab, "mid.attn.0", ch[L - 1], cfg.mid_depth, cfg.ctx_dim, &gather);
  u.mid_res1 = add_resblock(tab, "mid.res.1", ch[L - 1], ch[L - 1], cfg.temb_dim);
  c_prev = ch[L - 1];
  for (int up = 0; up < L; ++up) {
    const int l = L - 1 - up;
    UNetW::UpLevel lv;
    for (int i = 0; i <= cfg.layers_per_block; ++i) {
      const int cs = skips.back();
      skips.pop_back();
      const std::string p = "up." + std::to_string(up);
      lv.res.push_back(add_resblock(tab, p + ".res." + std::to_string(i), c_prev + cs, ch[l], cfg.temb_dim));
      c_prev = ch[l];
      if (cfg.attn_depth[l] > 0)
        lv.attn.push_back(
            add_transformer(tab, p + ".attn." + std::to_string(i), ch[l], cfg.attn_depth[l], cfg.ctx_dim, &gather));
    }
    lv.has_up = up < L - 1;
    if (lv.has_up) lv.up = add_conv3x3(tab, "up." + std::to_string(up) + ".up", ch[l], ch[l]);
    u.up.push_back(lv);
  }
  u.out = add_output(tab, ch[0], cfg.out_channels);
  if (!gather.k.empty()) {
    // [K of every cross-attention | V of every cross-attention], one row per output feature
    u.ctx_kv_w = tab.place_run(gather.k);
    tab.place_run(gather.v);
    u.ctx_k_cols = gather.cols;
  }
  return u;
}

static ResW add_vae_resblock(Table& tab, const std::string& p, int ci, int co) {
  ResW w;
  w.c_in = ci;
  w.c_out = co;
  w.n1g = tab.add(p + ".norm1.gamma", {ci}, SD_KIND_NORM_GAMMA, 0);
  w.n1b = tab.add(p + ".norm1.beta", {ci}, SD_KIND_NORM_BETA, 0);
  w.c1w = tab.add(p + ".conv1.weight", {co, ci, 3, 3}, SD_KIND_WEIGHT, ci * 9, PACK_CONV_KRSC);
  w.c1b = tab.add(p + ".conv1.bias", {co}, SD_KIND_BIAS, ci * 9);
  w.tw = w.tb = -1;
  w.n2g = tab.add(p + ".norm2.gamma", {co}, SD_KIND_NORM_GAMMA, 0);
  w.n2b = tab.add(p + ".norm2.beta", {co}, SD_KIND_NORM_BETA, 0);
  w.c2w = tab.add(p + ".conv2.weight", {co, co, 3, 3}, SD_KIND_WEIGHT, co * 9, PACK_CONV_KRSC);
  w.c2b = tab.add(p + ".conv2.bias", {co}, SD_KIND_BIAS, co * 9);
  w.sw = w.sb = -1;
  if (ci != co) {
    w.sw = tab.add(p + ".skip.weight", {co, ci, 1, 1}, SD_KIND_WEIGHT, ci);
    w.sb = tab.add(p + ".skip.bias", {co}, SD_KIND_BIAS, ci);
  }
  return w;
}

VaeW add_vae(Table& tab, const sd_vae_cfg& cfg) {
  VaeW v;
  const int L = cfg.n_levels;
  const int lc = cfg.latent_channels;
  std::vector<int> ch;
  for (int l = L - 1; l >= 0; --l) ch.push_back(cfg.block_channels[l]);
  v.post_quant.w = tab.add("post_quant_conv.weight", {lc, lc, 1, 1}, SD_KIND_WEIGHT, lc);
  v.post_quant.b = tab.add("post_quant_conv.bias", {lc}, SD_KIND_BIAS, lc);
  v.conv_in_kp = conv_in_kp(lc);
  v.conv_in = add_conv_in(tab, "conv_in", lc, ch[0], v.conv_in_kp);
  v.mid_res0 = add_vae_resblock(tab, "mid.res.0", ch[0], ch[0]);
  {
    const int C = ch[0];
    VaeAttnW& a = v.mid_attn;
    a.C = C;
    a.ng = tab.add("mid.attn.norm.gamma", {C}, SD_KIND_NORM_GAMMA, 0);
    a.nb = tab.add("mid.attn.norm.beta", {C}, SD_KIND_NORM_BETA, 0);
    // q, k, v weights consecutive (each a multiple of 256 bytes): one [3C, C] matrix; same for the biases
    a.qkv = tab.add("mid.attn.q.weight", {C, C}, SD_KIND_WEIGHT, C);
    tab.add("mid.attn.k.weight", {C, C}, SD_KIND_WEIGHT, C);
    tab.add("mid.attn.v.weight", {C, C}, SD_KIND_WEIGHT, C);
    a.qkv_b = tab.add("mid.attn.q.bias", {C}, SD_KIND_BIAS, C);
    tab.add("mid.attn.k.bias", {C}, SD_KIND_BIAS, C);
    tab.add("mid.attn.v.bias", {C}, SD_KIND_BIAS, C);
    a.ow = tab.add("mid.attn.out.weight", {C, C}, SD_KIND_WEIGHT, C);
    a.ob = tab.add("mid.attn.out.bias", {C}, SD_KIND_BIAS, C);
  }
  v.mid_res1 = add_vae_resblock(tab, "mid.res.1", ch[0], ch[0]);
  int c_prev = ch[0];
  for (int i = 0; i < L; ++i) {
    VaeW::Level lv;
    lv.C = ch[i];
    for (int j = 0; j <= cfg.layers_per_block; ++j) {
      lv.res.push_back(add_vae_resblock(tab, "up." + std::to_string(i) + ".res." + std::to_string(j), c_prev, ch[i]));
      c_prev = ch[i];
    }
    lv.has_up = i < L - 1;
    if (lv.has_up) lv.up = add_conv3x3(tab, "up." + std::to_string(i) + ".up", ch[i], ch[i]);
    v.up.push_back(lv);
  }
  v.out = add_output(tab, ch[L - 1], cfg.out_channels);
  return v;
}

namespace {

float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

// Round to nearest even; inputs here are finite products of two BF16 values.
uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

// Canonical row of packed row r of a (possibly GEGLU-interleaved) [rows][K] matrix.
int64_t canon_row(int64_t r, int64_t rows, bool geglu) {
  if (!geglu) return r;
  return (r & 1) ? rows / 2 + (r >> 1) : (r >> 1);
}

}  // namespace

void pack(const Table& tab, const uint16_t* canon, uint8_t* packed) {
  memset(packed, 0, (size_t)tab.packed_bytes);
  for (const Tensor& x : tab.t) {
    const uint16_t* src = canon + x.canon_off;
    uint16_t* dst = reinterpret_cast<uint16_t*>(packed + x.packed_off);
    const int64_t n = x.numel();
    switch (x.pack) {
      case PACK_COPY:
        memcpy(dst, src, (size_t)n * 2);
        break;
      case PACK_CONV_KRSC: {
        const int64_t O = x.shape[0], C = x.shape[1], KH = x.shape[2], KW = x.shape[3];
        for (int64_t o = 0; o < O; ++o)
          for (int64_t c = 0; c < C; ++c)
            for (int64_t u = 0; u < KH; ++u)
              for (int64_t v = 0; v < KW; ++v)
                dst[((o * KH + u) * KW + v) * C + c] = src[((o * C + c) * KH + u) * KW + v];
        break;
      }
      case PACK_CONV_IM2COL: {
        const int64_t O = x.shape[0], C = x.shape[1], Kp = x.aux;
        for (int64_t o = 0; o < O; ++o)
          for (int64_t c = 0; c < C; ++c)
            for (int64_t t = 0; t < 9; ++t) dst[o * Kp + t * C + c] = src[(o * C + c) * 9 + t];
        break;
      }
      case PACK_GEGLU_ROWS: {
        const int64_t R = x.shape[0], K = x.shape[1], half = R / 2;
        for (int64_t j = 0; j < half; ++j) {
          memcpy(dst + (2 * j) * K, src + j * K, (size_t)K * 2);
          memcpy(dst + (2 * j + 1) * K, src + (half + j) * K, (size_t)K * 2);
        }
        break;
      }
      case PACK_GEGLU_BIAS: {
        const int64_t half = x.shape[0] / 2;
        for (int64_t j = 0; j < half; ++j) {
          dst[2 * j] = src[j];
          dst[2 * j + 1] = src[half + j];
        }
        break;
      }
      case PACK_LNFOLD:
      case PACK_LNFOLD_GEGLU: {
        const uint16_t* gamma = canon + tab.t[x.aux].canon_off;
        const int64_t R = x.shape[0], K = x.shape[1];
        const bool geglu = x.pack == PACK_LNFOLD_GEGLU;
        for (int64_t r = 0; r < R; ++r) {
          const uint16_t* row = src + canon_row(r, R, geglu) * K;
          for (int64_t k = 0; k < K; ++k) dst[r * K + k] = f32_to_bf16(bf16_to_f32(row[k]) * bf16_to_f32(gamma[k]));
        }
        break;
      }
    }
  }
  // derived column terms (after every tensor: c1 reads the packed W')
  for (const Derived& x : tab.d) {
    float* out = reinterpret_cast<float*>(packed + x.out_off);
    const Tensor& wt = tab.t[x.w_tensor];
    if (!x.c2) {
      const uint16_t* wp = reinterpret_cast<const uint16_t*>(packed + wt.packed_off);
      for (int64_t r = 0; r < x.rows; ++r) {
        double s = 0;
        for (int64_t k = 0; k < x.K; ++k) s += bf16_to_f32(wp[r * x.K + k]);
        out[r] = (float)s;
      }
    } else {
      const uint16_t* wc = canon + wt.canon_off;
      const uint16_t* beta = canon + tab.t[x.beta_tensor].canon_off;
      const uint16_t* bias = x.bias_tensor >= 0 ? canon + tab.t[x.bias_tensor].canon_off : nullptr;
      for (int64_t r = 0; r < x.rows; ++r) {
        const int64_t cr = canon_row(r, x.rows, x.geglu);
        double s = bias ? bf16_to_f32(bias[cr]) : 0.0;
        for (int64_t k = 0; k < x.K; ++k) s += (double)bf16_to_f32(wc[cr * x.K + k]) * bf16_to_f32(beta[k]);
        out[r] = (float)s;
      }
    }
  }
}

sd_status export_table(const Table& tab, sd_tensor_desc* out, int32_t capacity, int32_t* n_tensors,
                       int64_t* canon_elems, int64_t* packed_bytes) {
  if (n_tensors) *n_tensors = (int32_t)tab.t.size();
  if (canon_elems) *canon_elems = tab.canon_elems;
  if (packed_bytes) *packed_bytes = tab.packed_bytes;
  if (!out) return SD_OK;
  if (capacity < (int32_t)tab.t.size()) return SD_ERR_CAPACITY;
  for (size_t i = 0; i < tab.t.size(); ++i) {
    const Tensor& x = tab.t[i];
    sd_tensor_desc& d = out[i];
    memset(&d, 0, sizeof(d));
    strncpy(d.name, x.name.c_str(), sizeof(d.name) - 1);
    d.ndim = x.ndim;
    for (int k = 0; k < 4; ++k) d.shape[k] = x.shape[k];
    d.kind = x.kind;
    d.fan_in = x.fan_in;
    d.canon_offset = x.canon_off;
    d.packed_offset = x.packed_off;
  }
  return SD_OK;
}

}  // namespace sdw
