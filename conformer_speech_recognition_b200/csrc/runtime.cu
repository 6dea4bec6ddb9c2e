// Host runtime behind include/gam.h: argument checks, weight validation and
// repacking, one preallocated workspace per context, per-call length planning
// (segment layout, see common.cuh), the launch sequence of the encoder and of
// the CTC decoder, launch counting / CUDA-event profiling and host-side fault
// injection.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <optional>
#include <string>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/gam.h"
#include "common.cuh"
#include "gemm_tc.cuh"

using namespace gam;

namespace {

// An NVTX range for the lifetime of the object (one per stage of the path), so a
// timeline tool shows frontend / subsampling / each block / the heads by name.
// Header-only NVTX: without an attached tool each call is a no-op.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local std::string g_create_error;

const char* kKindNames[PK_COUNT] = {"frontend",  "gemm_subsampling", "gemm_ffn_up",  "gemm_ffn_down",
                                    "gemm_qkv",  "gemm_attn_out",    "gemm_pw1_glu", "gemm_pw2",
                                    "attention", "layernorm",        "dwconv",       "ctc_gemm",
                                    "ctc_softmax_argmax", "ctc_collapse", "misc", "rnnt_enc_proj",
                                    "rnnt_decode"};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Lengths of one clip (see gam.h).
struct ClipLen {
  int F, T1, T2, L1, L2;
};
ClipLen clip_len(int64_t n, const gam_config& c) {
  ClipLen r{0, 0, 0, 0, 0};
  if (n < c.win) return r;
  r.F = (int)(1 + (n - c.win) / c.hop);
  const int k = c.sub_kernel, p = k / 2;
  r.T1 = (r.F + 2 * p - k) / 2 + 1;
  r.T2 = (r.T1 + 2 * p - k) / 2 + 1;
  r.L1 = (r.F - 1) / 2;
  r.L2 = r.L1 >= 1 ? (r.L1 - 1) / 2 : 0;
  return r;
}
// Encoder rows reserved for a clip of F frames (segment layout).
int seg_rows(const ClipLen& l) {
  int64_t a = ceil_div(l.F + 2, 4), b = ceil_div(l.L1 + 2, 2), c = l.L2 + 1;
  return (int)round_up(std::max(a, std::max(b, c)), 8);
}

struct DevLinear {
  void* w = nullptr;          // [N, K] f32 / f16 / int8, or packed 6- / 4-bit rows (see upload_linear)
  __half* scale = nullptr;    // int8: [N, K/64]
  __half* scale_t = nullptr;  // int8: [K/64, N]
  float* b = nullptr;         // [N]
  int N = 0, K = 0, dtype = 0;  // dtype: 0 f32, 1 f16, 2 int8, 3 int6, 4 int4 (g64 scales)
  WeightOp op() const { return WeightOp{w, scale, dtype, scale_t}; }
};
struct DevLN {
  float* g = nullptr;
  float* b = nullptr;
};
struct DevLayer {
  DevLN ln_ffn1, ln_attn, ln_conv, ln_ffn2, ln_out;
  DevLinear ffn1_up, ffn1_down, qkv, out, pw1, pw2, ffn2_up, ffn2_down;
  float* dw_w = nullptr;  // [K][d], BatchNorm folded
  float* dw_b = nullptr;  // [d]
};

// RNNT head (gam_rnnt_attach): the joint's encoder projection as a GEMM weight,
// the LSTM input-gate table per symbol and transposed fp16 weights of the
// sequential part.
struct RnntHead {
  int C = 0, P = 0, E = 0, J = 0, max_symbols = 0, act = 0;
  DevLinear enc;            // fp16 modes: [W_enc | W_enc] rows padded to 256, K = 2d; fp32 mode: W_enc
  float* gtab = nullptr;    // [(C + 1)][4P]
  __half* whh = nullptr;    // [4P][P]
  __half* wp = nullptr;     // [J][P]
  float* bp = nullptr;      // [J]
  __half* wo = nullptr;     // [C][J]
  float* bo = nullptr;      // [C]
  float* eproj = nullptr;   // [max_batch * T2_cap][J]
};

struct Prof {
  uint32_t mask = 0;  // families whose launches are timed
  int64_t launches[PK_COUNT] = {};
  double ms[PK_COUNT] = {};
  std::vector<cudaEvent_t> ev;  // event pair i = (ev[2i], ev[2i+1])
  std::vector<int> pair_kind;   // family of pair i (-1: recording failed)
  int npairs = 0;               // pairs recorded since the last read
};

constexpr int kRing = 8;

// CUDA graphs for repeated calls.  A call is identified by everything its
// kernel sequence depends on besides buffer contents: the entry point, the
// clip lengths (hence the plan and every launch shape) and the caller's
// pointers.  The first call with a key runs eagerly; the second is captured
// (on a private stream) into a graph that reads the call's clip table from one
// of kGraphCap table slots preallocated with the context, and every later call
// replays it with one cudaGraphLaunch.  A slot's table is uploaded with an
// asynchronous copy on the caller's stream (from the pinned ring), after the
// last replay of the slot's previous graph (an event recorded at each launch),
// so capture and eviction neither allocate nor synchronise.
struct GraphEntry {
  std::vector<int64_t> key;
  cudaGraphExec_t exec = nullptr;
  int slot = -1;         // table slot: the captured kernels read c->graph_tables + slot * stride
  uint64_t used = 0;
};
struct GraphCache {
  bool enabled = true;
  cudaStream_t cap = nullptr;
  std::vector<GraphEntry> entries;
  std::vector<std::vector<int64_t>> seen;  // keys met once
  uint64_t tick = 0;
};
constexpr size_t kGraphCap = 16, kSeenCap = 64;

}  // namespace

struct gam_ctx {
  gam_config cfg{};
  int device = 0;
  int act_half = 0;  // activations between GEMMs in fp16 (1) or fp32 (0)
  int wdtype = 0;    // GEMM weight dtype: 0 f32, 1 f16, 2 int8-g64, 3 int6-g64, 4 int4-g64
  int d_head = 0;
  std::string err;
  std::vector<void*> allocs;
  // weights
  float* basis = nullptr;  // [320][320]
  float* fb = nullptr;     // [161][64]
  int* fb_range = nullptr; // [64][2]: first and last nonzero filterbank row of each mel bin
  // fp16 / INT8 modes: windowed DFT basis [384][320] as tf32 hi and lo parts, rows
  // [cos 64 bins | sin 64 bins] per 128 (bins 0 .. 191, zero past 160)
  float* dft_hi = nullptr;
  float* dft_lo = nullptr;
  float* split_hi = nullptr;  // [R0_cap + 2][160] packed samples, tf32 hi / lo parts
  float* split_lo = nullptr;
  DevLinear conv1, conv2, head;
  DevLinear head2;         // tensor-core CTC head: [W | W] padded to a multiple of 256 rows, K = 2d
  __half* ctc_a = nullptr; // [rows, 2d] fp16 hi / lo split of the valid encoder frames
  std::vector<DevLayer> layers;
  float* rope_cos = nullptr;  // [T2_cap][d_head/2]
  float* rope_sin = nullptr;
  // capacity
  int F_cap = 0, T2_cap = 0;
  int64_t E_cap = 0, R1_cap = 0, R0_cap = 0;
  // workspace
  void* mel = nullptr;
  void* c1 = nullptr;
  float* x = nullptr;
  void* u = nullptr;
  void* urot = nullptr;
  void* g = nullptr;
  void* h = nullptr;
  void* qk = nullptr;
  void* vt = nullptr;
  float* logits = nullptr;
  int* argmax = nullptr;
  float* audio_stage = nullptr;
  float* enc_stage = nullptr;
  int* tokens_stage = nullptr;
  int* counts_stage = nullptr;
  int* dev_status = nullptr;
  // per-call table ring (pinned host -> device)
  int* tab_host[kRing] = {};
  int* tab_dev[kRing] = {};
  cudaEvent_t tab_ev[kRing] = {};
  int ring = 0;
  size_t tab_ints = 0;  // ints per table (ring entries and graph slots)
  // graph table slots [kGraphCap][tab_ints] and, per slot, an event recorded after
  // every launch of the graph that reads it
  int* graph_tables = nullptr;
  cudaEvent_t graph_ev[kGraphCap] = {};
  cudaStream_t last_stream = nullptr;
  // tcgen05 GEMM plans
  TcGemmCache tc;
  RnntHead rnnt;
  Prof prof;
  GraphCache graphs;
  int inject_err = 0, inject_count = 0;
};

// Pseudo-streaming state (gam_stream_*): the last `window` samples of the audio
// pushed so far, in one of two device buffers (each push writes the new window
// into the other one, so in steady state the encoder sees two alternating
// pointers and its CUDA graphs replay), plus the per-step outputs.
struct gam_stream {
  gam_ctx* ctx = nullptr;
  int64_t window = 0;   // samples kept (at most 30 s at 16 kHz by default)
  int64_t len = 0;      // samples in the current window
  int64_t total = 0;    // samples pushed since the last reset
  int cur = 0;          // buffer holding the window
  float* buf[2] = {nullptr, nullptr};
  float* enc = nullptr;    // [1][T'(window)][d]
  int32_t* tok = nullptr;  // [T'(window)]
  int32_t* cnt = nullptr;  // [1]
  int t_cap = 0;
  int32_t* tok_host = nullptr;  // pinned [T'(window) + 1]
  std::vector<void*> allocs;
};

namespace {

gam_status fail(gam_ctx* c, gam_status s, const std::string& msg) {
  if (c) c->err = msg;
  else g_create_error = msg;
  return s;
}

gam_status cuda_check(gam_ctx* c, cudaError_t e, const char* what) {
  if (c && c->inject_count > 0) {
    c->inject_count--;
    e = (cudaError_t)c->inject_err;
  }
  if (e == cudaSuccess) return GAM_OK;
  return fail(c, GAM_ERR_CUDA, std::string(what) + ": " + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
}

#define GAM_TRY(expr)                  \
  do {                                 \
    gam_status _s = (expr);            \
    if (_s != GAM_OK) return _s;       \
  } while (0)

template <class F>
gam_status run_kernel(gam_ctx* c, int kind, cudaStream_t s, F&& launch) {
  Prof& p = c->prof;
  p.launches[kind]++;
  int slot = -1;
  if (((p.mask >> kind) & 1u) && p.npairs < (int)p.pair_kind.size()) {
    slot = p.npairs++;
    p.pair_kind[slot] = cudaEventRecord(p.ev[2 * slot], s) == cudaSuccess ? kind : -1;
  }
  const cudaError_t e = launch();
  if (slot >= 0 && cudaEventRecord(p.ev[2 * slot + 1], s) != cudaSuccess) p.pair_kind[slot] = -1;
  return cuda_check(c, e, kKindNames[kind]);
}

gam_status dev_alloc(gam_ctx* c, void** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) return cuda_check(c, e, "cudaMalloc");
  c->allocs.push_back(*p);
  return GAM_OK;
}
template <class T>
gam_status upload(gam_ctx* c, T** dst, const void* src, size_t bytes) {
  GAM_TRY(dev_alloc(c, (void**)dst, bytes));
  return cuda_check(c, cudaMemcpy(*dst, src, bytes, cudaMemcpyHostToDevice), "cudaMemcpy weights");
}

// ---- weight table ----
struct WeightTable {
  std::map<std::string, const gam_tensor*> by_name;
};

// shape entries of -1 accept any positive extent of at most max_free (when max_free > 0)
gam_status find(gam_ctx* c, const WeightTable& t, const std::string& name, std::vector<int64_t> shape,
                const gam_tensor** out, bool allow_trailing_one = false, int64_t max_free = 0) {
  auto it = t.by_name.find(name);
  if (it == t.by_name.end()) return fail(c, GAM_ERR_WEIGHTS, "missing tensor " + name);
  const gam_tensor* g = it->second;
  std::vector<int64_t> got(g->shape, g->shape + std::max(0, std::min(g->ndim, 4)));
  if (allow_trailing_one && got.size() == shape.size() + 1 && got.back() == 1) got.pop_back();
  bool free_ok = got.size() == shape.size();
  for (size_t i = 0; free_ok && i < shape.size(); ++i)
    if (shape[i] == -1) {
      free_ok = got[i] >= 1 && (max_free <= 0 || got[i] <= max_free);
      shape[i] = got[i];
    }
  if (!free_ok || got != shape || g->data == nullptr) {
    std::string s = "tensor " + name + " has shape [";
    for (auto v : got) s += std::to_string(v) + ",";
    s += "], expected [";
    for (auto v : shape) s += std::to_string(v) + ",";
    return fail(c, GAM_ERR_WEIGHTS, s + "]");
  }
  *out = g;
  return GAM_OK;
}

// Reads a float tensor (f32 or f16) into doubles.
gam_status read_f(gam_ctx* c, const gam_tensor* g, std::vector<double>& v) {
  int64_t n = 1;
  for (int i = 0; i < g->ndim; ++i) n *= g->shape[i];
  v.resize(n);
  if (g->dtype == GAM_DTYPE_F32) {
    const float* p = (const float*)g->data;
    for (int64_t i = 0; i < n; ++i) v[i] = p[i];
  } else if (g->dtype == GAM_DTYPE_F16) {
    const __half* p = (const __half*)g->data;
    for (int64_t i = 0; i < n; ++i) v[i] = (double)__half2float(p[i]);
  } else {
    return fail(c, GAM_ERR_WEIGHTS, std::string("tensor ") + g->name + " must be f32 or f16");
  }
  return GAM_OK;
}

gam_status get_vec(gam_ctx* c, const WeightTable& t, const std::string& name, int64_t n, std::vector<double>& v) {
  const gam_tensor* g;
  GAM_TRY(find(c, t, name, {n}, &g));
  return read_f(c, g, v);
}

gam_status upload_f32(gam_ctx* c, float** dst, const std::vector<double>& v) {
  std::vector<float> f(v.begin(), v.end());
  return upload(c, dst, f.data(), f.size() * sizeof(float));
}

gam_status load_ln(gam_ctx* c, const WeightTable& t, const std::string& name, int d, DevLN& ln) {
  std::vector<double> g, b;
  GAM_TRY(get_vec(c, t, name + ".weight", d, g));
  GAM_TRY(get_vec(c, t, name + ".bias", d, b));
  GAM_TRY(upload_f32(c, &ln.g, g));
  return upload_f32(c, &ln.b, b);
}

// Host copy of a linear weight in its device format, rows possibly permuted.
struct HostLinear {
  int N = 0, K = 0, dtype = 0;
  std::vector<double> w;        // f32 / f16 modes: [N, K] values
  std::vector<int8_t> q;        // quantised modes: [N, K] integer values
  std::vector<__half> s;        // quantised modes: [N, K/64] group scales
  std::vector<double> b;
};

gam_status read_linear(gam_ctx* c, const WeightTable& t, const std::string& name, int N, int K, bool quantized,
                       HostLinear& out) {
  out.N = N;
  out.K = K;
  GAM_TRY(get_vec(c, t, name + ".bias", N, out.b));
  if (quantized) {
    const gam_tensor *gq, *gs;
    GAM_TRY(find(c, t, name + ".weight_q", {N, K}, &gq, true));
    GAM_TRY(find(c, t, name + ".weight_scale", {N, K / 64}, &gs));
    if (gq->dtype != GAM_DTYPE_I8 || gs->dtype != GAM_DTYPE_F16)
      return fail(c, GAM_ERR_WEIGHTS, name + ": weight_q must be int8 and weight_scale f16");
    out.dtype = c->wdtype;
    out.q.assign((const int8_t*)gq->data, (const int8_t*)gq->data + (size_t)N * K);
    const int qmax = c->wdtype == 2 ? 127 : c->wdtype == 3 ? 31 : 7;
    for (int8_t v : out.q)
      if (v < -qmax || v > qmax)
        return fail(c, GAM_ERR_WEIGHTS, name + ".weight_q holds " + std::to_string((int)v) + ", outside +-" +
                                            std::to_string(qmax) + " of this precision");
    out.s.assign((const __half*)gs->data, (const __half*)gs->data + (size_t)N * (K / 64));
    return GAM_OK;
  }
  const gam_tensor* gw;
  GAM_TRY(find(c, t, name + ".weight", {N, K}, &gw, true));
  out.dtype = c->wdtype == 0 ? 0 : 1;
  return read_f(c, gw, out.w);
}

// Row permutation: new row i takes old row perm[i].
void permute_rows(HostLinear& l, const std::vector<int>& perm) {
  HostLinear o = l;
  for (int i = 0; i < l.N; ++i) {
    const int j = perm[i];
    o.b[i] = l.b[j];
    if (l.dtype >= 2) {
      std::memcpy(&o.q[(size_t)i * l.K], &l.q[(size_t)j * l.K], l.K);
      std::memcpy(&o.s[(size_t)i * (l.K / 64)], &l.s[(size_t)j * (l.K / 64)], (l.K / 64) * sizeof(__half));
    } else {
      std::memcpy(&o.w[(size_t)i * l.K], &l.w[(size_t)j * l.K], l.K * sizeof(double));
    }
  }
  l = std::move(o);
}

// 6- and 4-bit weights, stored as u = q + 32 (q + 8), packed per 16 consecutive
// weights v0 .. v15 of a row into the layout the GEMM's converter warps read
// (gemm_tc.cu): word w0 = low nibbles of v0 .. v7 with v_2i in nibble i and
// v_2i+1 in nibble 4 + i, word w1 the same for v8 .. v15, and for 6 bits a word
// w2 with the top two bits of v_2p in bits 2p .. 2p+1 and of v_2p+1 in bits
// 16 + 2p ..  Rows of K * bits / 8 bytes, chunks in K order.
void pack_subbyte(const HostLinear& l, std::vector<uint8_t>& out) {
  const bool six = l.dtype == 3;
  const int off = six ? 32 : 8, words = six ? 3 : 2;
  const size_t row_bytes = (size_t)l.K * (six ? 6 : 4) / 8;
  out.assign((size_t)l.N * row_bytes, 0);
  for (int n = 0; n < l.N; ++n)
    for (int c0 = 0; c0 < l.K; c0 += 16) {
      uint32_t w[3] = {0, 0, 0};
      for (int j = 0; j < 16; ++j) {
        const uint32_t u = (uint32_t)(l.q[(size_t)n * l.K + c0 + j] + off);
        const int jj = j & 7, p = j >> 1;
        const int nib = (jj & 1) ? 4 + (jj >> 1) : (jj >> 1);
        w[j >> 3] |= (u & 15u) << (4 * nib);
        if (six) w[2] |= (u >> 4) << ((j & 1) ? 16 + 2 * p : 2 * p);
      }
      std::memcpy(&out[(size_t)n * row_bytes + (size_t)(c0 / 16) * 4 * words], w, 4 * words);
    }
}

gam_status upload_linear(gam_ctx* c, const HostLinear& l, DevLinear& d) {
  d.N = l.N;
  d.K = l.K;
  d.dtype = l.dtype;
  GAM_TRY(upload_f32(c, &d.b, l.b));
  if (l.dtype >= 2) {
    if (l.dtype == 2) {
      GAM_TRY(upload(c, (int8_t**)&d.w, l.q.data(), l.q.size()));
    } else {
      std::vector<uint8_t> packed;
      pack_subbyte(l, packed);
      GAM_TRY(upload(c, (uint8_t**)&d.w, packed.data(), packed.size()));
    }
    const int G = l.K / 64;
    std::vector<__half> st((size_t)G * l.N);
    for (int n = 0; n < l.N; ++n)
      for (int g = 0; g < G; ++g) st[(size_t)g * l.N + n] = l.s[(size_t)n * G + g];
    GAM_TRY(upload(c, &d.scale_t, st.data(), st.size() * sizeof(__half)));
    return upload(c, &d.scale, l.s.data(), l.s.size() * sizeof(__half));
  }
  if (l.dtype == 0) {
    std::vector<float> f(l.w.begin(), l.w.end());
    return upload(c, (float**)&d.w, f.data(), f.size() * sizeof(float));
  }
  std::vector<__half> h(l.w.size());
  for (size_t i = 0; i < h.size(); ++i) h[i] = __float2half_rn((float)l.w[i]);
  return upload(c, (__half**)&d.w, h.data(), h.size() * sizeof(__half));
}

// Conv1d [out, in, K] -> GEMM weight [out, K * in] (tap-major rows).
gam_status load_conv(gam_ctx* c, const WeightTable& t, const std::string& name, int cout, int cin, int k,
                     DevLinear& d) {
  const gam_tensor* gw;
  GAM_TRY(find(c, t, name + ".weight", {cout, cin, k}, &gw));
  std::vector<double> w;
  GAM_TRY(read_f(c, gw, w));
  HostLinear l;
  l.N = cout;
  l.K = cin * k;
  l.dtype = c->wdtype == 0 ? 0 : 1;
  l.w.resize((size_t)cout * cin * k);
  for (int o = 0; o < cout; ++o)
    for (int ci = 0; ci < cin; ++ci)
      for (int kk = 0; kk < k; ++kk)
        l.w[((size_t)o * k + kk) * cin + ci] = w[((size_t)o * cin + ci) * k + kk];
  GAM_TRY(get_vec(c, t, name + ".bias", cout, l.b));
  return upload_linear(c, l, d);
}

// Nearest tf32 value of x (10 explicit mantissa bits; ties away from zero), as fp32.
float tf32_round(float x) {
  uint32_t u;
  std::memcpy(&u, &x, 4);
  if ((u & 0x7f800000u) != 0x7f800000u) {  // finite: round the magnitude at bit 13
    u += 0x1000u;
    u &= 0xffffe000u;
  }
  std::memcpy(&x, &u, 4);
  return x;
}

gam_status validate_config(const gam_config* cfg) {
  if (!cfg) return fail(nullptr, GAM_ERR_INVALID_ARG, "null config");
  const gam_config& c = *cfg;
  if (c.n_fft != 320 || c.win != 320 || c.hop != 160 || c.n_mels != 64)
    return fail(nullptr, GAM_ERR_INVALID_ARG, "frontend must be n_fft = win = 320, hop = 160, n_mels = 64");
  if (c.sub_kernel != 5) return fail(nullptr, GAM_ERR_INVALID_ARG, "sub_kernel must be 5");
  if (c.n_layers < 1 || c.d_model <= 0 || c.d_model % 256 || c.d_model > 1024)
    return fail(nullptr, GAM_ERR_INVALID_ARG, "d_model must be a multiple of 256, at most 1024");
  if (c.n_heads <= 0 || c.d_model % c.n_heads ||
      (c.d_model / c.n_heads != 48 && c.d_model / c.n_heads != 64))
    return fail(nullptr, GAM_ERR_INVALID_ARG, "d_model / n_heads must be 48 or 64");
  if (c.ffn_dim <= 0 || c.ffn_dim % 256) return fail(nullptr, GAM_ERR_INVALID_ARG, "ffn_dim must be a multiple of 256");
  if (c.conv_kernel < 1 || c.conv_kernel > 63 || c.conv_kernel % 2 == 0)
    return fail(nullptr, GAM_ERR_INVALID_ARG, "conv_kernel must be odd and <= 63");
  if (c.n_classes < 2 || c.n_classes > 1024) return fail(nullptr, GAM_ERR_INVALID_ARG, "n_classes must be 2..1024");
  if (c.precision < GAM_FP32 || c.precision > GAM_INT4_G64) return fail(nullptr, GAM_ERR_INVALID_ARG, "bad precision");
  if (!(c.rope_base > 0) || !(c.ln_eps > 0) || !(c.bn_eps > 0))
    return fail(nullptr, GAM_ERR_INVALID_ARG, "rope_base / eps must be positive");
  if (c.max_batch < 1 || c.max_batch > 4096) return fail(nullptr, GAM_ERR_INVALID_ARG, "max_batch must be 1..4096");
  if (c.max_samples < 1280 || c.max_samples > (int64_t)16000 * 3600)
    return fail(nullptr, GAM_ERR_INVALID_ARG, "max_samples must be 1280 .. 1 hour");
  return GAM_OK;
}

// Per-call plan.
struct Plan {
  int B = 0;
  std::vector<ClipLen> len;
  std::vector<int> e;  // B + 1
  int E = 0, E_pad = 0, R1 = 0, R0 = 0, F_max = 0, T2_max = 0;
};

gam_status make_plan(gam_ctx* c, const gam_config& cfg, const int32_t* lengths, int batch, int64_t max_samples,
                     Plan& p) {
  if (!lengths || batch < 1) return fail(c, GAM_ERR_INVALID_ARG, "lengths must be non-null and batch >= 1");
  p.B = batch;
  p.len.resize(batch);
  p.e.assign(batch + 1, 0);
  for (int i = 0; i < batch; ++i) {
    if (lengths[i] < 1280)
      return fail(c, GAM_ERR_SHAPE, "clip " + std::to_string(i) + " has " + std::to_string(lengths[i]) +
                                        " samples; at least 1280 are needed for one encoder frame");
    if (max_samples > 0 && lengths[i] > max_samples)
      return fail(c, GAM_ERR_SHAPE, "clip " + std::to_string(i) + " is longer than max_samples");
    p.len[i] = clip_len(lengths[i], cfg);
    p.e[i + 1] = p.e[i] + seg_rows(p.len[i]);
    p.F_max = std::max(p.F_max, p.len[i].F);
    p.T2_max = std::max(p.T2_max, p.len[i].T2);
  }
  p.E = p.e[batch];
  p.E_pad = (int)round_up(p.E, 128);
  p.R1 = (int)round_up(2 * (int64_t)p.E_pad + 4, 128);
  p.R0 = 2 * p.R1 + 4;
  return GAM_OK;
}

// The clip table read by the kernels (Clips): segment starts e[0..B], then F, L1,
// L2 and a zero row, B + 1 ints each.
int table_ints(const Plan& p) { return 5 * (p.B + 1); }
void fill_table(const Plan& p, int* h) {
  const int B = p.B;
  for (int i = 0; i <= B; ++i) h[i] = p.e[i];
  for (int i = 0; i < B; ++i) {
    h[(B + 1) + i] = p.len[i].F;
    h[2 * (B + 1) + i] = p.len[i].L1;
    h[3 * (B + 1) + i] = p.len[i].L2;
    h[4 * (B + 1) + i] = 0;
  }
}

// Upload the clip table (and optional extra ints) through the pinned ring.
gam_status upload_table(gam_ctx* c, const Plan& p, cudaStream_t s, Clips* out) {
  const int slot = c->ring;
  c->ring = (c->ring + 1) % kRing;
  GAM_TRY(cuda_check(c, cudaEventSynchronize(c->tab_ev[slot]), "ring event"));
  int* h = c->tab_host[slot];
  const int B = p.B;
  fill_table(p, h);
  const size_t bytes = table_ints(p) * sizeof(int);
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(c->tab_dev[slot], h, bytes, cudaMemcpyHostToDevice, s), "table upload"));
  GAM_TRY(cuda_check(c, cudaEventRecord(c->tab_ev[slot], s), "ring event record"));
  *out = Clips{c->tab_dev[slot], B};
  return GAM_OK;
}

gam_status upload_ints(gam_ctx* c, const int32_t* src, int n, cudaStream_t s, const int** out) {
  if (n < 0 || (size_t)n > c->tab_ints) return fail(c, GAM_ERR_CAPACITY, "table larger than a ring entry");
  const int slot = c->ring;
  c->ring = (c->ring + 1) % kRing;
  GAM_TRY(cuda_check(c, cudaEventSynchronize(c->tab_ev[slot]), "ring event"));
  std::memcpy(c->tab_host[slot], src, n * sizeof(int));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(c->tab_dev[slot], c->tab_host[slot], n * sizeof(int), cudaMemcpyHostToDevice, s),
                     "lengths upload"));
  GAM_TRY(cuda_check(c, cudaEventRecord(c->tab_ev[slot], s), "ring event record"));
  *out = c->tab_dev[slot];
  return GAM_OK;
}

// ---- CUDA graphs ----
bool graphs_usable(const gam_ctx* c) { return c->graphs.enabled && c->prof.mask == 0 && c->inject_count == 0; }

GraphEntry* graph_find(gam_ctx* c, const std::vector<int64_t>& key) {
  for (GraphEntry& e : c->graphs.entries)
    if (e.key == key) {
      e.used = ++c->graphs.tick;
      return &e;
    }
  return nullptr;
}

// True on the second call with this key (capture now); the first call only records it.
bool graph_second_sighting(gam_ctx* c, const std::vector<int64_t>& key) {
  auto& seen = c->graphs.seen;
  for (size_t i = 0; i < seen.size(); ++i)
    if (seen[i] == key) {
      seen.erase(seen.begin() + i);
      return true;
    }
  if (seen.size() >= kSeenCap) seen.erase(seen.begin());
  seen.push_back(key);
  return false;
}

// An executable graph still in flight is freed by the driver when it completes.
void graph_free(GraphEntry& e) {
  if (e.exec) cudaGraphExecDestroy(e.exec);
  e.exec = nullptr;
}

// Replay a cached graph on stream s and mark its table slot as in use until then.
gam_status graph_launch(gam_ctx* c, GraphEntry* e, cudaStream_t s) {
  GAM_TRY(cuda_check(c, cudaGraphLaunch(e->exec, s), "graph launch"));
  return cuda_check(c, cudaEventRecord(c->graph_ev[e->slot], s), "graph event");
}

// Capture body(device table, capture stream) into a graph for key.  The graph
// reads the call's table (table_host, n ints) from a preallocated slot: a free
// one, else the least recently used entry's (that entry is dropped).  The table
// is copied into the slot on stream s once the slot's last replay is done, so the
// graph's first launch on s sees it.  On success *out is the new cache entry.
template <class F>
gam_status graph_capture(gam_ctx* c, const std::vector<int64_t>& key, const int* table_host, int n, F&& body,
                         cudaStream_t s, GraphEntry** out) {
  GraphCache& gc = c->graphs;
  if ((size_t)n > c->tab_ints) return fail(c, GAM_ERR_CAPACITY, "clip table larger than its graph slot");
  int slot = -1;
  if (gc.entries.size() < kGraphCap) {
    std::vector<bool> used(kGraphCap, false);
    for (const GraphEntry& e : gc.entries) used[e.slot] = true;
    for (size_t i = 0; i < kGraphCap && slot < 0; ++i)
      if (!used[i]) slot = (int)i;
  } else {
    auto lru = std::min_element(gc.entries.begin(), gc.entries.end(),
                                [](const GraphEntry& a, const GraphEntry& b) { return a.used < b.used; });
    slot = lru->slot;
    graph_free(*lru);
    gc.entries.erase(lru);
  }
  int* table = c->graph_tables + (size_t)slot * c->tab_ints;
  // the pinned ring entry holds the table until the copy has run
  const int r = c->ring;
  c->ring = (c->ring + 1) % kRing;
  GAM_TRY(cuda_check(c, cudaEventSynchronize(c->tab_ev[r]), "ring event"));
  std::memcpy(c->tab_host[r], table_host, (size_t)n * sizeof(int));
  GAM_TRY(cuda_check(c, cudaStreamWaitEvent(s, c->graph_ev[slot], 0), "slot wait"));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(table, c->tab_host[r], (size_t)n * sizeof(int), cudaMemcpyHostToDevice, s),
                     "graph table upload"));
  GAM_TRY(cuda_check(c, cudaEventRecord(c->tab_ev[r], s), "ring event record"));
  GraphEntry e;
  e.key = key;
  e.slot = slot;
  cudaGraph_t g = nullptr;
  gam_status st = cuda_check(c, cudaStreamBeginCapture(gc.cap, cudaStreamCaptureModeThreadLocal), "capture");
  if (st == GAM_OK) {
    st = body(table, gc.cap);
    const gam_status end = cuda_check(c, cudaStreamEndCapture(gc.cap, &g), "end capture");
    if (st == GAM_OK) st = end;
  }
  if (st == GAM_OK) st = cuda_check(c, cudaGraphInstantiate(&e.exec, g, 0), "graph instantiate");
  if (g) cudaGraphDestroy(g);
  if (st != GAM_OK) {
    graph_free(e);
    return st;
  }
  e.used = ++gc.tick;
  gc.entries.push_back(e);
  *out = &gc.entries.back();
  return GAM_OK;
}

// ---- GEMM dispatch: tensor cores for fp16 / int8, CUDA cores for fp32 ----
gam_status gemm(gam_ctx* c, int kind, cudaStream_t s, const void* A, const void* A2, int n_split, int lda,
                const DevLinear& W, int M, int epi, float alpha, void* out, int ldo, const Clips& clips,
                int a_f32 = 0, int n_valid = 0) {
  EpiParams ep{};
  ep.out = out;
  ep.x = (float*)out;
  ep.bias = W.b;
  ep.alpha = alpha;
  ep.ldo = ldo;
  ep.clips = clips;
  ep.qk = c->qk;
  ep.vt = c->vt;
  ep.rows_pad = (int)c->E_cap;
  ep.n_heads = c->cfg.n_heads;
  ep.d_head = c->d_head;
  ep.d_model = c->cfg.d_model;
  ep.n_valid = n_valid ? n_valid : W.N;
  const int a_dtype = a_f32 ? 0 : (c->act_half ? 1 : 0);
  if (tc_supported(a_dtype, W.dtype, W.N, W.K, epi)) {
    return run_kernel(c, kind, s, [&] {
      return launch_gemm_tc(&c->tc, A, A2, n_split, lda, W.op(), M, W.N, W.K, epi, ep, s);
    });
  }
  return run_kernel(c, kind, s, [&] {
    return launch_gemm_simt(a_dtype, A, A2, n_split, lda, W.op(), M, W.N, W.K, epi, c->act_half, ep, s);
  });
}

gam_status encoder_kernels(gam_ctx* c, const Plan& p, const Clips& clips, const float* audio, int64_t max_samples,
                           int stop_layer, int stop_stage, float* out, cudaStream_t s);

// The encoder up to (layer, stage); stage < 0 runs everything.  Leaves the
// residual stream in c->x and scatters it to out.  Repeated identical calls
// replay a CUDA graph (see GraphCache).
gam_status run_encoder(gam_ctx* c, const float* audio, const int32_t* lengths, int batch, int64_t max_samples,
                       int stop_layer, int stop_stage, float* out, int32_t* enc_len_out, cudaStream_t s) {
  const gam_config& cfg = c->cfg;
  Plan p;
  GAM_TRY(make_plan(c, cfg, lengths, batch, max_samples, p));
  if (batch > cfg.max_batch) return fail(c, GAM_ERR_CAPACITY, "batch above max_batch");
  if (max_samples > cfg.max_samples) return fail(c, GAM_ERR_CAPACITY, "max_samples above the context's capacity");
  if (p.E_pad > c->E_cap || p.R1 > c->R1_cap || p.R0 > c->R0_cap || p.T2_max > c->T2_cap)
    return fail(c, GAM_ERR_CAPACITY, "workspace too small for this batch");
  if (!audio || !out) return fail(c, GAM_ERR_INVALID_ARG, "null audio or output pointer");
  c->last_stream = s;
  if (enc_len_out)
    for (int i = 0; i < batch; ++i) enc_len_out[i] = p.len[i].L2;
  if (graphs_usable(c)) {
    std::vector<int64_t> key = {0, stop_layer, stop_stage, (int64_t)(uintptr_t)audio, max_samples,
                                (int64_t)(uintptr_t)out, batch};
    key.insert(key.end(), lengths, lengths + batch);
    GraphEntry* e = graph_find(c, key);
    if (!e && graph_second_sighting(c, key)) {
      std::vector<int> tab(table_ints(p));
      fill_table(p, tab.data());
      GAM_TRY(graph_capture(c, key, tab.data(), (int)tab.size(), [&](const int* t, cudaStream_t cs) {
        return encoder_kernels(c, p, Clips{t, batch}, audio, max_samples, stop_layer, stop_stage, out, cs);
      }, s, &e));
    }
    if (e) return graph_launch(c, e, s);
  }
  Clips clips;
  GAM_TRY(upload_table(c, p, s, &clips));
  return encoder_kernels(c, p, clips, audio, max_samples, stop_layer, stop_stage, out, s);
}

// The encoder's kernel sequence for plan p (table already on the device).
gam_status encoder_kernels(gam_ctx* c, const Plan& p, const Clips& clips, const float* audio, int64_t max_samples,
                           int stop_layer, int stop_stage, float* out, cudaStream_t s) {
  const gam_config& cfg = c->cfg;
  const int d = cfg.d_model, f = cfg.ffn_dim, H = cfg.n_heads, dh = c->d_head;
  const int ah = c->act_half;
  const float eps = cfg.ln_eps;
  const int M = p.E_pad;

  std::optional<NvtxRange> stage_range;
  stage_range.emplace("gam.frontend");
  if (c->dft_hi) {
    // tensor-core frontend: samples split into tf32 hi / lo rows, then the 3xTF32 DFT
    // with power, filterbank and log in its epilogue (fp16 packed mel rows)
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_audio_split(audio, max_samples, clips, p.R0 + 1, c->split_hi, c->split_lo, s);
    }));
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_dft_mel(&c->tc, c->split_hi, c->split_lo, p.R0 + 1, c->dft_hi, c->dft_lo, c->fb, c->fb_range,
                            clips, p.R0, 0, 0, c->mel, s);
    }));
  } else {
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_frontend(audio, max_samples, clips, p.R0, 1, 0, c->basis, c->fb, c->mel, ah, s);
    }));
  }
  stage_range.reset();
  stage_range.emplace("gam.subsampling");
  GAM_TRY(gemm(c, PK_GEMM_SUB, s, c->mel, nullptr, 0, 2 * cfg.n_mels, c->conv1, p.R1, EPI_CONV1, 1.f, c->c1, d,
               clips));
  GAM_TRY(gemm(c, PK_GEMM_SUB, s, c->c1, nullptr, 0, 2 * d, c->conv2, M, EPI_CONV2, 1.f, c->x, d, clips));

  const int L = cfg.n_layers;
  bool stopped = stop_stage == GAM_STAGE_SUBSAMPLING;
  stage_range.reset();
  static const char* const kLayerNames[] = {
      "gam.layer.0",  "gam.layer.1",  "gam.layer.2",  "gam.layer.3",  "gam.layer.4",  "gam.layer.5",
      "gam.layer.6",  "gam.layer.7",  "gam.layer.8",  "gam.layer.9",  "gam.layer.10", "gam.layer.11",
      "gam.layer.12", "gam.layer.13", "gam.layer.14", "gam.layer.15", "gam.layer.16", "gam.layer.17",
      "gam.layer.18", "gam.layer.19", "gam.layer.20", "gam.layer.21", "gam.layer.22", "gam.layer.23"};
  for (int l = 0; l < L && !stopped; ++l) {
    NvtxRange layer_range(l < 24 ? kLayerNames[l] : "gam.layer");
    DevLayer& w = c->layers[l];
    if (l == 0)
      GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
        return launch_layernorm(c->x, w.ln_ffn1.g, w.ln_ffn1.b, eps, c->u, ah, M, d, s);
      }));
    // FFN1 (half-step residual)
    GAM_TRY(gemm(c, PK_GEMM_FFN_UP, s, c->u, nullptr, 0, d, w.ffn1_up, M, EPI_SWISH, 1.f, c->h, f, clips));
    GAM_TRY(gemm(c, PK_GEMM_FFN_DOWN, s, c->h, nullptr, 0, f, w.ffn1_down, M, EPI_RESID, 0.5f, c->x, d, clips));
    if (l == stop_layer && stop_stage == GAM_STAGE_FFN1) { stopped = true; break; }
    // rotary MHSA
    GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
      return launch_layernorm_rope(c->x, w.ln_attn.g, w.ln_attn.b, eps, c->rope_cos, c->rope_sin, clips, c->u,
                                   c->urot, ah, M, d, dh, s);
    }));
    GAM_TRY(gemm(c, PK_GEMM_QKV, s, c->urot, c->u, 2 * d, d, w.qkv, M, EPI_QKV, 1.f, nullptr, 0, clips));
    GAM_TRY(run_kernel(c, PK_ATTENTION, s, [&] {
      return launch_attention(&c->tc, c->qk, c->vt, clips, c->urot, ah, (int)c->E_cap, H, dh, p.T2_max, s);
    }));
    GAM_TRY(gemm(c, PK_GEMM_OUT, s, c->urot, nullptr, 0, d, w.out, M, EPI_RESID, 1.f, c->x, d, clips));
    if (l == stop_layer && stop_stage == GAM_STAGE_MHSA) { stopped = true; break; }
    // convolution module
    GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
      return launch_layernorm(c->x, w.ln_conv.g, w.ln_conv.b, eps, c->u, ah, M, d, s);
    }));
    GAM_TRY(gemm(c, PK_GEMM_PW1, s, c->u, nullptr, 0, d, w.pw1, M, EPI_GLU, 1.f, c->g, d, clips));
    GAM_TRY(run_kernel(c, PK_DWCONV, s, [&] {
      return launch_dwconv(c->g, w.dw_w, w.dw_b, clips, c->u, ah, M, d, cfg.conv_kernel, c->tc.sm_count,
                           c->tc.status, s);
    }));
    GAM_TRY(gemm(c, PK_GEMM_PW2, s, c->u, nullptr, 0, d, w.pw2, M, EPI_RESID, 1.f, c->x, d, clips));
    if (l == stop_layer && stop_stage == GAM_STAGE_CONV) { stopped = true; break; }
    // FFN2
    GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
      return launch_layernorm(c->x, w.ln_ffn2.g, w.ln_ffn2.b, eps, c->u, ah, M, d, s);
    }));
    GAM_TRY(gemm(c, PK_GEMM_FFN_UP, s, c->u, nullptr, 0, d, w.ffn2_up, M, EPI_SWISH, 1.f, c->h, f, clips));
    GAM_TRY(gemm(c, PK_GEMM_FFN_DOWN, s, c->h, nullptr, 0, f, w.ffn2_down, M, EPI_RESID, 0.5f, c->x, d, clips));
    if (l == stop_layer && stop_stage == GAM_STAGE_FFN2) { stopped = true; break; }
    // block-final LayerNorm, chained with the next block's first one
    const bool last = (l == L - 1) || (l == stop_layer && stop_stage == GAM_STAGE_LAYER);
    if (!last) {
      DevLayer& nx = c->layers[l + 1];
      GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
        return launch_layernorm_chain(c->x, w.ln_out.g, w.ln_out.b, nx.ln_ffn1.g, nx.ln_ffn1.b, eps, c->u, ah, M, d,
                                      s);
      }));
    } else {
      GAM_TRY(run_kernel(c, PK_LAYERNORM, s, [&] {
        return launch_layernorm(c->x, w.ln_out.g, w.ln_out.b, eps, c->x, 0, M, d, s);
      }));
      stopped = (l == stop_layer);
    }
  }
  return run_kernel(c, PK_MISC, s, [&] { return launch_scatter_out(c->x, clips, out, p.T2_max, d, s); });
}

gam_status ctc_kernels(gam_ctx* c, const float* enc, const int* lo, int batch, int t_max, int M_valid, float* logp,
                       int32_t* tokens, int32_t* counts, int32_t* frames, cudaStream_t s);

// CTC decoding of encoder output; repeated identical calls replay a CUDA graph.
gam_status run_ctc(gam_ctx* c, const float* enc, const int32_t* enc_len, int batch, int t_max, float* logp,
                   int32_t* tokens, int32_t* counts, cudaStream_t s, int32_t* frames = nullptr) {
  const gam_config& cfg = c->cfg;
  if (!enc || !enc_len || !tokens || !counts) return fail(c, GAM_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || t_max < 1) return fail(c, GAM_ERR_INVALID_ARG, "batch and t_max must be >= 1");
  if (batch > cfg.max_batch || t_max > c->T2_cap) return fail(c, GAM_ERR_CAPACITY, "batch or t_max above capacity");
  for (int i = 0; i < batch; ++i)
    if (enc_len[i] < 0 || enc_len[i] > t_max) return fail(c, GAM_ERR_SHAPE, "enc_len outside [0, t_max]");
  c->last_stream = s;
  // lengths and the offsets of the compacted valid frames, one upload
  std::vector<int32_t> lo(2 * batch + 1);
  for (int i = 0; i < batch; ++i) lo[i] = enc_len[i];
  lo[batch] = 0;
  for (int i = 0; i < batch; ++i) lo[batch + 1 + i] = lo[batch + i] + enc_len[i];
  if (graphs_usable(c)) {
    std::vector<int64_t> key = {1, (int64_t)(uintptr_t)enc, batch, t_max, (int64_t)(uintptr_t)logp,
                                (int64_t)(uintptr_t)tokens, (int64_t)(uintptr_t)counts, (int64_t)(uintptr_t)frames};
    key.insert(key.end(), enc_len, enc_len + batch);
    GraphEntry* e = graph_find(c, key);
    if (!e && graph_second_sighting(c, key)) {
      GAM_TRY(graph_capture(c, key, lo.data(), (int)lo.size(), [&](const int* t, cudaStream_t cs) {
        return ctc_kernels(c, enc, t, batch, t_max, lo[2 * batch], logp, tokens, counts, frames, cs);
      }, s, &e));
    }
    if (e) return graph_launch(c, e, s);
  }
  const int* dev;
  GAM_TRY(upload_ints(c, lo.data(), 2 * batch + 1, s, &dev));
  return ctc_kernels(c, enc, dev, batch, t_max, lo[2 * batch], logp, tokens, counts, frames, s);
}

// CTC head, log-softmax / argmax and collapse; lo = [enc_len (batch) | offsets of the
// compacted valid frames (batch + 1)] on the device, M_valid = total valid frames.
gam_status ctc_kernels(gam_ctx* c, const float* enc, const int* lo, int batch, int t_max, int M_valid, float* logp,
                       int32_t* tokens, int32_t* counts, int32_t* frames, cudaStream_t s) {
  NvtxRange range("gam.ctc");
  const gam_config& cfg = c->cfg;
  const int* lens = lo;
  const int* off = lo + batch;
  const int C = cfg.n_classes, M = batch * t_max;
  Clips none{nullptr, 0};
  if (c->head2.w) {
    // tensor cores: logits = [hi | lo] . [W | W]^T on the valid frames only
    if (M_valid > 0) {
      GAM_TRY(run_kernel(c, PK_CTC_GEMM, s, [&] {
        return launch_split_hi_lo(enc, off, batch, t_max, cfg.d_model, M_valid, c->ctc_a, s);
      }));
      GAM_TRY(gemm(c, PK_CTC_GEMM, s, c->ctc_a, nullptr, 0, 2 * cfg.d_model, c->head2, M_valid, EPI_F32, 1.f,
                   c->logits, C, none, 0, C));
    }
    GAM_TRY(run_kernel(c, PK_CTC_SOFTMAX, s, [&] {
      return launch_logsoftmax_argmax(c->logits, C, lens, batch, t_max, C, logp, c->argmax, s, off);
    }));
  } else {
    GAM_TRY(gemm(c, PK_CTC_GEMM, s, enc, nullptr, 0, cfg.d_model, c->head, M, EPI_F32, 1.f, c->logits, C, none, 1));
    GAM_TRY(run_kernel(c, PK_CTC_SOFTMAX, s, [&] {
      return launch_logsoftmax_argmax(c->logits, C, lens, batch, t_max, C, logp, c->argmax, s);
    }));
  }
  return run_kernel(c, PK_CTC_COLLAPSE, s, [&] {
    return launch_collapse(c->argmax, lens, batch, t_max, C - 1, tokens, counts, s, frames);
  });
}

gam_status build_weights(gam_ctx* c, const gam_tensor* tensors, int n) {
  const gam_config& cfg = c->cfg;
  WeightTable t;
  for (int i = 0; i < n; ++i) {
    if (!tensors[i].name) return fail(c, GAM_ERR_WEIGHTS, "tensor without a name");
    t.by_name[tensors[i].name] = &tensors[i];
  }
  const int d = cfg.d_model, f = cfg.ffn_dim, K = cfg.conv_kernel;
  const bool q8 = cfg.precision >= GAM_INT8_G64;  // quantised linear weights (8, 6 or 4 bits)
  // frontend: window folded into the DFT basis
  {
    std::vector<double> win, fbv;
    GAM_TRY(get_vec(c, t, "frontend.window", cfg.win, win));
    const gam_tensor* g;
    GAM_TRY(find(c, t, "frontend.mel_fb", {cfg.n_fft / 2 + 1, cfg.n_mels}, &g));
    GAM_TRY(read_f(c, g, fbv));
    const int N = cfg.n_fft;
    std::vector<double> basis((size_t)N * N, 0.0);
    const double two_pi = 6.283185307179586476925286766559;
    for (int nn = 0; nn < N; ++nn)
      for (int k = 0; k <= N / 2; ++k) {
        const double a = two_pi * (double)((int64_t)k * nn % N) / N;
        basis[(size_t)nn * N + k] = win[nn] * std::cos(a);
        if (k >= 1 && k < N / 2) basis[(size_t)nn * N + N / 2 + k] = win[nn] * std::sin(a);
      }
    GAM_TRY(upload_f32(c, &c->basis, basis));
    GAM_TRY(upload_f32(c, &c->fb, fbv));
    {
      const int nb = cfg.n_fft / 2 + 1, nm = cfg.n_mels;
      std::vector<int> range(2 * (size_t)nm);
      for (int m = 0; m < nm; ++m) {
        int lo = nb, hi = -1;
        for (int k = 0; k < nb; ++k)
          if ((float)fbv[(size_t)k * nm + m] != 0.f) {
            lo = std::min(lo, k);
            hi = k;
          }
        range[2 * m] = hi < 0 ? 0 : lo;
        range[2 * m + 1] = hi;
      }
      GAM_TRY(upload(c, &c->fb_range, range.data(), range.size() * sizeof(int)));
    }
    if (cfg.precision != GAM_FP32) {
      // tensor-core DFT basis: row n = [cos | sin] block n / 128, bin 64 (n / 128) + n % 64,
      // each value as tf32 hi + lo (lo = the remainder, itself rounded to tf32)
      const int rows = 384;
      std::vector<float> bh((size_t)rows * N, 0.f), bl((size_t)rows * N, 0.f);
      for (int row = 0; row < rows; ++row) {
        const int within = row % 128;
        const bool is_sin = within >= 64;
        const int bin = (row / 128) * 64 + (within % 64);
        if (bin > N / 2 || (is_sin && (bin == 0 || bin == N / 2))) continue;
        for (int nn = 0; nn < N; ++nn) {
          const double a = two_pi * (double)((int64_t)bin * nn % N) / N;
          const double v = win[nn] * (is_sin ? std::sin(a) : std::cos(a));
          const float hi = tf32_round((float)v);
          bh[(size_t)row * N + nn] = hi;
          bl[(size_t)row * N + nn] = tf32_round((float)(v - (double)hi));
        }
      }
      GAM_TRY(upload(c, &c->dft_hi, bh.data(), bh.size() * sizeof(float)));
      GAM_TRY(upload(c, &c->dft_lo, bl.data(), bl.size() * sizeof(float)));
    }
  }
  GAM_TRY(load_conv(c, t, "subsampling.conv1", d, cfg.n_mels, cfg.sub_kernel, c->conv1));
  GAM_TRY(load_conv(c, t, "subsampling.conv2", d, d, cfg.sub_kernel, c->conv2));
  c->layers.resize(cfg.n_layers);
  for (int l = 0; l < cfg.n_layers; ++l) {
    const std::string p = "layers." + std::to_string(l) + ".";
    DevLayer& w = c->layers[l];
    GAM_TRY(load_ln(c, t, p + "ffn1.norm", d, w.ln_ffn1));
    GAM_TRY(load_ln(c, t, p + "attn.norm", d, w.ln_attn));
    GAM_TRY(load_ln(c, t, p + "conv.norm", d, w.ln_conv));
    GAM_TRY(load_ln(c, t, p + "ffn2.norm", d, w.ln_ffn2));
    GAM_TRY(load_ln(c, t, p + "norm_out", d, w.ln_out));
    HostLinear hl;
    GAM_TRY(read_linear(c, t, p + "ffn1.linear1", f, d, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.ffn1_up));
    GAM_TRY(read_linear(c, t, p + "ffn1.linear2", d, f, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.ffn1_down));
    GAM_TRY(read_linear(c, t, p + "ffn2.linear1", f, d, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.ffn2_up));
    GAM_TRY(read_linear(c, t, p + "ffn2.linear2", d, f, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.ffn2_down));
    // Q, K, V concatenated along the output dim
    {
      HostLinear q, k, v;
      GAM_TRY(read_linear(c, t, p + "attn.linear_q", d, d, q8, q));
      GAM_TRY(read_linear(c, t, p + "attn.linear_k", d, d, q8, k));
      GAM_TRY(read_linear(c, t, p + "attn.linear_v", d, d, q8, v));
      HostLinear all = q;
      all.N = 3 * d;
      all.b.insert(all.b.end(), k.b.begin(), k.b.end());
      all.b.insert(all.b.end(), v.b.begin(), v.b.end());
      if (q8) {
        all.q.insert(all.q.end(), k.q.begin(), k.q.end());
        all.q.insert(all.q.end(), v.q.begin(), v.q.end());
        all.s.insert(all.s.end(), k.s.begin(), k.s.end());
        all.s.insert(all.s.end(), v.s.begin(), v.s.end());
      } else {
        all.w.insert(all.w.end(), k.w.begin(), k.w.end());
        all.w.insert(all.w.end(), v.w.begin(), v.w.end());
      }
      GAM_TRY(upload_linear(c, all, w.qkv));
    }
    GAM_TRY(read_linear(c, t, p + "attn.linear_out", d, d, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.out));
    // pointwise1: interleave value / gate rows in blocks of 64 for the GLU epilogue
    GAM_TRY(read_linear(c, t, p + "conv.pointwise1", 2 * d, d, q8, hl));
    {
      std::vector<int> perm(2 * d);
      for (int i = 0; i < 2 * d; ++i) {
        const int blk = i / 128, within = i % 128;
        perm[i] = within < 64 ? blk * 64 + within : d + blk * 64 + (within - 64);
      }
      permute_rows(hl, perm);
    }
    GAM_TRY(upload_linear(c, hl, w.pw1));
    GAM_TRY(read_linear(c, t, p + "conv.pointwise2", d, d, q8, hl));
    GAM_TRY(upload_linear(c, hl, w.pw2));
    // depthwise + BatchNorm folded: y = s * (sum w x + b - mean) + beta, s = gamma / sqrt(var + eps)
    {
      const gam_tensor* gw;
      GAM_TRY(find(c, t, p + "conv.depthwise.weight", {d, 1, K}, &gw));
      std::vector<double> dw, db, gm, bt, mu, var;
      GAM_TRY(read_f(c, gw, dw));
      GAM_TRY(get_vec(c, t, p + "conv.depthwise.bias", d, db));
      GAM_TRY(get_vec(c, t, p + "conv.bn.weight", d, gm));
      GAM_TRY(get_vec(c, t, p + "conv.bn.bias", d, bt));
      GAM_TRY(get_vec(c, t, p + "conv.bn.running_mean", d, mu));
      GAM_TRY(get_vec(c, t, p + "conv.bn.running_var", d, var));
      std::vector<double> wf((size_t)K * d), bf(d);
      for (int ch = 0; ch < d; ++ch) {
        const double sc = gm[ch] / std::sqrt(var[ch] + (double)cfg.bn_eps);
        for (int k = 0; k < K; ++k) wf[(size_t)k * d + ch] = dw[(size_t)ch * K + k] * sc;
        bf[ch] = (db[ch] - mu[ch]) * sc + bt[ch];
      }
      GAM_TRY(upload_f32(c, &w.dw_w, wf));
      GAM_TRY(upload_f32(c, &w.dw_b, bf));
    }
  }
  {
    HostLinear hl;
    GAM_TRY(read_linear(c, t, "head", cfg.n_classes, d, q8, hl));
    GAM_TRY(upload_linear(c, hl, c->head));
    if (cfg.precision != GAM_FP32) {
      // [W | W] with zero rows up to a multiple of 256: one fp16 tensor-core GEMM of
      // the hi / lo split activations gives fp32-grade logits
      const int Cp = (int)round_up(cfg.n_classes, 256);
      HostLinear h2;
      h2.N = Cp;
      h2.K = 2 * d;
      h2.dtype = hl.dtype;
      h2.b.assign(Cp, 0.0);
      for (int n = 0; n < cfg.n_classes; ++n) h2.b[n] = hl.b[n];
      if (hl.dtype >= 2) {
        h2.q.assign((size_t)Cp * 2 * d, 0);
        h2.s.assign((size_t)Cp * (2 * d / 64), __float2half(1.f));
        const int G = d / 64;
        for (int n = 0; n < cfg.n_classes; ++n) {
          for (int h = 0; h < 2; ++h) {
            std::memcpy(&h2.q[(size_t)n * 2 * d + h * d], &hl.q[(size_t)n * d], d);
            for (int g = 0; g < G; ++g) h2.s[(size_t)n * 2 * G + h * G + g] = hl.s[(size_t)n * G + g];
          }
        }
      } else {
        h2.w.assign((size_t)Cp * 2 * d, 0.0);
        for (int n = 0; n < cfg.n_classes; ++n)
          for (int h = 0; h < 2; ++h)
            std::memcpy(&h2.w[(size_t)n * 2 * d + h * d], &hl.w[(size_t)n * d], d * sizeof(double));
      }
      GAM_TRY(upload_linear(c, h2, c->head2));
    }
  }
  // RoPE tables, base rope_base, positions 0 .. T2_cap - 1
  {
    const int half = c->d_head / 2;
    std::vector<double> cs((size_t)c->T2_cap * half), sn((size_t)c->T2_cap * half);
    for (int tt = 0; tt < c->T2_cap; ++tt)
      for (int i = 0; i < half; ++i) {
        const double inv = std::pow((double)cfg.rope_base, -2.0 * i / c->d_head);
        cs[(size_t)tt * half + i] = std::cos(tt * inv);
        sn[(size_t)tt * half + i] = std::sin(tt * inv);
      }
    GAM_TRY(upload_f32(c, &c->rope_cos, cs));
    GAM_TRY(upload_f32(c, &c->rope_sin, sn));
  }
  return GAM_OK;
}

gam_status alloc_workspace(gam_ctx* c) {
  const gam_config& cfg = c->cfg;
  ClipLen lmax = clip_len(cfg.max_samples, cfg);
  c->F_cap = lmax.F;
  c->T2_cap = lmax.T2;
  c->E_cap = round_up((int64_t)cfg.max_batch * seg_rows(lmax), 128);
  c->R1_cap = round_up(2 * c->E_cap + 4, 128);
  c->R0_cap = 2 * c->R1_cap + 4;
  const size_t es = c->act_half ? 2 : 4;
  const int d = cfg.d_model, f = cfg.ffn_dim, H = cfg.n_heads;
  const int64_t E = c->E_cap;
  GAM_TRY(dev_alloc(c, &c->mel, (size_t)c->R0_cap * cfg.n_mels * es));
  if (cfg.precision != GAM_FP32) {
    GAM_TRY(dev_alloc(c, (void**)&c->split_hi, (size_t)(c->R0_cap + 2) * cfg.hop * 4));
    GAM_TRY(dev_alloc(c, (void**)&c->split_lo, (size_t)(c->R0_cap + 2) * cfg.hop * 4));
  }
  GAM_TRY(dev_alloc(c, &c->c1, (size_t)c->R1_cap * d * es));
  GAM_TRY(dev_alloc(c, (void**)&c->x, (size_t)E * d * 4));
  GAM_TRY(dev_alloc(c, &c->u, (size_t)E * d * es));
  GAM_TRY(dev_alloc(c, &c->urot, (size_t)E * d * es));
  GAM_TRY(dev_alloc(c, &c->g, (size_t)E * d * es));
  GAM_TRY(dev_alloc(c, &c->h, (size_t)E * f * es));
  GAM_TRY(dev_alloc(c, &c->qk, (size_t)2 * H * E * 64 * es));
  GAM_TRY(dev_alloc(c, &c->vt, (size_t)H * 64 * E * es));
  const int64_t ctc_rows = (int64_t)cfg.max_batch * c->T2_cap;
  GAM_TRY(dev_alloc(c, (void**)&c->logits, (size_t)ctc_rows * cfg.n_classes * 4));
  GAM_TRY(dev_alloc(c, (void**)&c->argmax, (size_t)ctc_rows * 4));
  if (cfg.precision != GAM_FP32) GAM_TRY(dev_alloc(c, (void**)&c->ctc_a, (size_t)ctc_rows * 2 * cfg.d_model * 2));
  GAM_TRY(dev_alloc(c, (void**)&c->audio_stage, (size_t)cfg.max_batch * cfg.max_samples * 4));
  GAM_TRY(dev_alloc(c, (void**)&c->enc_stage, (size_t)ctc_rows * d * 4));
  GAM_TRY(dev_alloc(c, (void**)&c->tokens_stage, (size_t)ctc_rows * 4));
  GAM_TRY(dev_alloc(c, (void**)&c->counts_stage, (size_t)cfg.max_batch * 4));
  GAM_TRY(dev_alloc(c, (void**)&c->dev_status, 16));
  // zero once: the padded head-dim columns and every buffer read before written
  GAM_TRY(cuda_check(c, cudaMemset(c->qk, 0, (size_t)2 * H * E * 64 * es), "memset"));
  GAM_TRY(cuda_check(c, cudaMemset(c->vt, 0, (size_t)H * 64 * E * es), "memset"));
  GAM_TRY(cuda_check(c, cudaMemset(c->dev_status, 0, 16), "memset"));
  const size_t tab_ints = 5 * (size_t)(cfg.max_batch + 1) + 16;  // also >= 3 * max_batch + 1
  c->tab_ints = tab_ints;
  for (int i = 0; i < kRing; ++i) {
    GAM_TRY(cuda_check(c, cudaMallocHost((void**)&c->tab_host[i], tab_ints * 4), "cudaMallocHost"));
    GAM_TRY(dev_alloc(c, (void**)&c->tab_dev[i], tab_ints * 4));
    GAM_TRY(cuda_check(c, cudaEventCreateWithFlags(&c->tab_ev[i], cudaEventDisableTiming), "event"));
  }
  // CUDA-graph table slots, their events and the private capture stream
  GAM_TRY(dev_alloc(c, (void**)&c->graph_tables, kGraphCap * tab_ints * 4));
  for (size_t i = 0; i < kGraphCap; ++i)
    GAM_TRY(cuda_check(c, cudaEventCreateWithFlags(&c->graph_ev[i], cudaEventDisableTiming), "event"));
  GAM_TRY(cuda_check(c, cudaStreamCreateWithFlags(&c->graphs.cap, cudaStreamNonBlocking), "capture stream"));
  c->prof.ev.resize(2 * 16384);
  c->prof.pair_kind.assign(16384, -1);
  for (auto& e : c->prof.ev) GAM_TRY(cuda_check(c, cudaEventCreate(&e), "event"));
  return GAM_OK;
}

void destroy(gam_ctx* c) {
  if (!c) return;
  cudaSetDevice(c->device);
  cudaDeviceSynchronize();
  tc_release(&c->tc);
  for (void* p : c->allocs) cudaFree(p);
  for (int i = 0; i < kRing; ++i) {
    if (c->tab_host[i]) cudaFreeHost(c->tab_host[i]);
    if (c->tab_ev[i]) cudaEventDestroy(c->tab_ev[i]);
  }
  for (auto& e : c->prof.ev)
    if (e) cudaEventDestroy(e);
  for (GraphEntry& e : c->graphs.entries) graph_free(e);
  for (size_t i = 0; i < kGraphCap; ++i)
    if (c->graph_ev[i]) cudaEventDestroy(c->graph_ev[i]);
  if (c->graphs.cap) cudaStreamDestroy(c->graphs.cap);
  delete c;
}

gam_status rnnt_attach(gam_ctx* c, const gam_rnnt_config& rc, const gam_tensor* tensors, int n) {
  const int d = c->cfg.d_model;
  const int C = rc.n_classes, P = rc.pred_dim, J = rc.joint_dim;
  if (C < 2 || C > 4096 || P < 8 || P > 1024 || P % 8 || J < 8 || J > 1024 || J % 8 || rc.max_symbols < 1 ||
      rc.max_symbols > 64 || (rc.joint_act != 0 && rc.joint_act != 1))
    return fail(c, GAM_ERR_INVALID_ARG, "rnnt config: n_classes 2..4096, pred_dim / joint_dim multiples of 8 up to "
                                        "1024, max_symbols 1..64, joint_act 0 or 1");
  if (rnnt_smem_bytes(C, P, J) > 200 * 1024) return fail(c, GAM_ERR_INVALID_ARG, "rnnt head too large");
  WeightTable t;
  for (int i = 0; i < n; ++i) {
    if (!tensors[i].name) return fail(c, GAM_ERR_WEIGHTS, "tensor without a name");
    t.by_name[tensors[i].name] = &tensors[i];
  }
  const gam_tensor* ge;
  GAM_TRY(find(c, t, "rnnt.embed.weight", {C, -1}, &ge, false, 4096));
  const int E = (int)ge->shape[1];
  std::vector<double> emb, wih, whh, bih, bhh, we, be, wp, bp, wo, bo;
  GAM_TRY(read_f(c, ge, emb));
  const gam_tensor* g;
  GAM_TRY(find(c, t, "rnnt.lstm.weight_ih_l0", {4 * P, E}, &g));
  GAM_TRY(read_f(c, g, wih));
  GAM_TRY(find(c, t, "rnnt.lstm.weight_hh_l0", {4 * P, P}, &g));
  GAM_TRY(read_f(c, g, whh));
  GAM_TRY(get_vec(c, t, "rnnt.lstm.bias_ih_l0", 4 * P, bih));
  GAM_TRY(get_vec(c, t, "rnnt.lstm.bias_hh_l0", 4 * P, bhh));
  GAM_TRY(find(c, t, "rnnt.joint.enc.weight", {J, d}, &g));
  GAM_TRY(read_f(c, g, we));
  GAM_TRY(get_vec(c, t, "rnnt.joint.enc.bias", J, be));
  GAM_TRY(find(c, t, "rnnt.joint.pred.weight", {J, P}, &g));
  GAM_TRY(read_f(c, g, wp));
  GAM_TRY(get_vec(c, t, "rnnt.joint.pred.bias", J, bp));
  GAM_TRY(find(c, t, "rnnt.joint.out.weight", {C, J}, &g));
  GAM_TRY(read_f(c, g, wo));
  GAM_TRY(get_vec(c, t, "rnnt.joint.out.bias", C, bo));
  RnntHead& r = c->rnnt;
  if (r.gtab) return fail(c, GAM_ERR_INVALID_ARG, "an RNNT head is attached already");
  // input gates per symbol, emb[k] W_ih^T + b_ih + b_hh (both biases), and the start row (zero input)
  std::vector<double> gt((size_t)(C + 1) * 4 * P);
  for (int k = 0; k <= C; ++k)
    for (int row = 0; row < 4 * P; ++row) {
      double v = bih[row] + bhh[row];
      if (k < C)
        for (int e = 0; e < E; ++e) v += emb[(size_t)k * E + e] * wih[(size_t)row * E + e];
      gt[(size_t)k * 4 * P + row] = v;
    }
  auto to_half = [](const std::vector<double>& w) {  // row-major, as given
    std::vector<__half> o(w.size());
    for (size_t i = 0; i < w.size(); ++i) o[i] = __float2half_rn((float)w[i]);
    return o;
  };
  std::vector<__half> whh_h = to_half(whh), wp_h = to_half(wp), wo_h = to_half(wo);
  GAM_TRY(upload_f32(c, &r.gtab, gt));
  GAM_TRY(upload(c, &r.whh, whh_h.data(), whh_h.size() * sizeof(__half)));
  GAM_TRY(upload(c, &r.wp, wp_h.data(), wp_h.size() * sizeof(__half)));
  GAM_TRY(upload_f32(c, &r.bp, bp));
  GAM_TRY(upload(c, &r.wo, wo_h.data(), wo_h.size() * sizeof(__half)));
  GAM_TRY(upload_f32(c, &r.bo, bo));
  HostLinear hl;
  if (c->cfg.precision == GAM_FP32) {
    hl.N = J;
    hl.K = d;
    hl.dtype = 0;
    hl.w = we;
    hl.b = be;
  } else {
    // [W | W] against the fp16 hi / lo split of the frames (as the CTC head): fp32-grade projection
    const int Np = (int)round_up(J, 256);
    hl.N = Np;
    hl.K = 2 * d;
    hl.dtype = 1;
    hl.b.assign(Np, 0.0);
    hl.w.assign((size_t)Np * 2 * d, 0.0);
    for (int j = 0; j < J; ++j) {
      hl.b[j] = be[j];
      for (int h = 0; h < 2; ++h)
        std::memcpy(&hl.w[(size_t)j * 2 * d + h * d], &we[(size_t)j * d], d * sizeof(double));
    }
  }
  GAM_TRY(upload_linear(c, hl, r.enc));
  GAM_TRY(dev_alloc(c, (void**)&r.eproj, (size_t)c->cfg.max_batch * c->T2_cap * J * 4));
  r.C = C;
  r.P = P;
  r.E = E;
  r.J = J;
  r.max_symbols = rc.max_symbols;
  r.act = rc.joint_act;
  return cuda_check(c, cudaDeviceSynchronize(), "rnnt attach sync");
}

gam_status rnnt_greedy(gam_ctx* c, const float* enc, const int32_t* enc_len, int batch, int t_max, int max_tokens,
                       int32_t* tokens, int32_t* frames, int32_t* counts, cudaStream_t s) {
  const gam_config& cfg = c->cfg;
  RnntHead& r = c->rnnt;
  if (!r.gtab) return fail(c, GAM_ERR_INVALID_ARG, "no RNNT head attached (gam_rnnt_attach)");
  if (!enc || !enc_len || !tokens || !counts) return fail(c, GAM_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || t_max < 1 || max_tokens < 1) return fail(c, GAM_ERR_INVALID_ARG, "batch, t_max, max_tokens >= 1");
  if (batch > cfg.max_batch || t_max > c->T2_cap) return fail(c, GAM_ERR_CAPACITY, "batch or t_max above capacity");
  for (int i = 0; i < batch; ++i)
    if (enc_len[i] < 0 || enc_len[i] > t_max) return fail(c, GAM_ERR_SHAPE, "enc_len outside [0, t_max]");
  c->last_stream = s;
  NvtxRange range("gam.rnnt");
  // lengths [B], first eproj rows [B + 1], clips by decreasing length [B]
  std::vector<int32_t> lo(3 * batch + 1);
  for (int i = 0; i < batch; ++i) lo[i] = enc_len[i];
  lo[batch] = 0;
  for (int i = 0; i < batch; ++i) lo[batch + 1 + i] = lo[batch + i] + enc_len[i];
  const int M_valid = lo[2 * batch];
  int32_t* order = lo.data() + 2 * batch + 1;
  for (int i = 0; i < batch; ++i) order[i] = i;
  std::stable_sort(order, order + batch, [&](int32_t x, int32_t y) { return enc_len[x] > enc_len[y]; });
  const int* dev;
  GAM_TRY(upload_ints(c, lo.data(), 3 * batch + 1, s, &dev));
  const int* lens = dev;
  const int* off = dev + batch;
  const int* ord = dev + 2 * batch + 1;
  Clips none{nullptr, 0};
  if (cfg.precision != GAM_FP32) {
    if (M_valid > 0) {
      GAM_TRY(run_kernel(c, PK_RNNT_ENC_PROJ, s, [&] {
        return launch_split_hi_lo(enc, off, batch, t_max, cfg.d_model, M_valid, c->ctc_a, s);
      }));
      GAM_TRY(gemm(c, PK_RNNT_ENC_PROJ, s, c->ctc_a, nullptr, 0, 2 * cfg.d_model, r.enc, M_valid, EPI_F32, 1.f,
                   r.eproj, r.J, none, 0, r.J));
    }
  } else {
    GAM_TRY(gemm(c, PK_RNNT_ENC_PROJ, s, enc, nullptr, 0, cfg.d_model, r.enc, batch * t_max, EPI_F32, 1.f, r.eproj,
                 r.J, none, 1));
    off = nullptr;  // rows b * t_max + t
  }
  return run_kernel(c, PK_RNNT_DECODE, s, [&] {
    return launch_rnnt_greedy(r.eproj, lens, off, ord, batch, t_max, r.gtab, r.whh, r.wp, r.bp, r.wo, r.bo, r.C, r.P,
                              r.J, r.max_symbols, r.act, max_tokens, tokens, frames, counts, c->tc.status, s);
  });
}

gam_status enter(gam_ctx* c) {
  if (!c) return GAM_ERR_INVALID_ARG;
  c->err.clear();
  return cuda_check(c, cudaSetDevice(c->device), "cudaSetDevice");
}

}  // namespace

void gam::set_context_free_error(const std::string& msg) { g_create_error = msg; }

bool gam::pdl_enabled() {
  static const bool on = [] {
    const char* v = std::getenv("GAM_PDL");
    return !(v && std::strcmp(v, "0") == 0);
  }();
  return on;
}

extern "C" {

const char* gam_status_string(gam_status s) {
  switch (s) {
    case GAM_OK: return "GAM_OK";
    case GAM_ERR_INVALID_ARG: return "GAM_ERR_INVALID_ARG";
    case GAM_ERR_SHAPE: return "GAM_ERR_SHAPE";
    case GAM_ERR_CAPACITY: return "GAM_ERR_CAPACITY";
    case GAM_ERR_WEIGHTS: return "GAM_ERR_WEIGHTS";
    case GAM_ERR_UNSUPPORTED_DEVICE: return "GAM_ERR_UNSUPPORTED_DEVICE";
    case GAM_ERR_CUDA: return "GAM_ERR_CUDA";
    case GAM_ERR_DEVICE_TIMEOUT: return "GAM_ERR_DEVICE_TIMEOUT";
  }
  return "GAM_ERR_UNKNOWN";
}

const char* gam_last_error(const gam_ctx* ctx) { return ctx ? ctx->err.c_str() : g_create_error.c_str(); }

gam_status gam_plan_lengths(const gam_config* cfg, const int32_t* lengths, int batch, int32_t* frames_out,
                            int32_t* enc_len_out, int32_t* dims_out) {
  g_create_error.clear();
  GAM_TRY(validate_config(cfg));
  Plan p;
  GAM_TRY(make_plan(nullptr, *cfg, lengths, batch, 0, p));
  for (int i = 0; i < batch; ++i) {
    if (frames_out) frames_out[i] = p.len[i].F;
    if (enc_len_out) enc_len_out[i] = p.len[i].L2;
  }
  if (dims_out) {
    dims_out[0] = p.F_max;
    dims_out[1] = p.T2_max;
  }
  return GAM_OK;
}

gam_status gam_create(const gam_config* cfg, const gam_tensor* tensors, int n_tensors, int device, gam_ctx** out) {
  g_create_error.clear();
  if (!out) return fail(nullptr, GAM_ERR_INVALID_ARG, "null output pointer");
  *out = nullptr;
  GAM_TRY(validate_config(cfg));
  if (!tensors || n_tensors <= 0) return fail(nullptr, GAM_ERR_INVALID_ARG, "no weight tensors");
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess || device < 0 || device >= ndev)
    return fail(nullptr, GAM_ERR_UNSUPPORTED_DEVICE, std::string("no CUDA device ") + std::to_string(device) + ": " +
                                                          cudaGetErrorString(e));
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, device) != cudaSuccess || prop.major != 10 || prop.minor != 0)
    return fail(nullptr, GAM_ERR_UNSUPPORTED_DEVICE, "device is not compute capability 10.0 (B200 / sm_100a)");
  gam_ctx* c = new gam_ctx();
  c->cfg = *cfg;
  c->device = device;
  c->act_half = cfg->precision == GAM_FP32 ? 0 : 1;
  c->wdtype = cfg->precision == GAM_FP32 ? 0 : (cfg->precision == GAM_FP16 ? 1 : cfg->precision);
  c->d_head = cfg->d_model / cfg->n_heads;
  if (const char* v = std::getenv("GAM_CUDA_GRAPHS")) c->graphs.enabled = std::strcmp(v, "0") != 0;
  gam_status s = cuda_check(c, cudaSetDevice(device), "cudaSetDevice");
  if (s == GAM_OK) s = cuda_check(c, tc_init(&c->tc, device), "tensor-core init");
  if (s == GAM_OK) s = alloc_workspace(c);
  if (s == GAM_OK) s = build_weights(c, tensors, n_tensors);
  if (s == GAM_OK) s = cuda_check(c, cudaDeviceSynchronize(), "create sync");
  if (s != GAM_OK) {
    g_create_error = c->err;
    destroy(c);
    return s;
  }
  *out = c;
  return GAM_OK;
}

gam_status gam_destroy(gam_ctx* ctx) {
  destroy(ctx);
  return GAM_OK;
}

gam_status gam_logmel(gam_ctx* c, const float* audio, const int32_t* lengths, int batch, int64_t max_samples,
                      float* mel, int32_t* frames_out, void* stream) {
  GAM_TRY(enter(c));
  if (!audio || !mel) return fail(c, GAM_ERR_INVALID_ARG, "null pointer");
  if (batch > c->cfg.max_batch) return fail(c, GAM_ERR_CAPACITY, "batch above max_batch");
  Plan p;
  GAM_TRY(make_plan(c, c->cfg, lengths, batch, max_samples, p));
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  Clips clips;
  if (c->dft_hi) {
    // the tensor-core frontend gam_encode runs, writing the padded fp32 output
    if (p.R0 > c->R0_cap) return fail(c, GAM_ERR_CAPACITY, "clips longer than the context's workspace");
    GAM_TRY(upload_table(c, p, s, &clips));
    GAM_TRY(cuda_check(c, cudaMemsetAsync(mel, 0, (size_t)batch * p.F_max * c->cfg.n_mels * 4, s), "memset"));
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_audio_split(audio, max_samples, clips, p.R0 + 1, c->split_hi, c->split_lo, s);
    }));
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_dft_mel(&c->tc, c->split_hi, c->split_lo, p.R0 + 1, c->dft_hi, c->dft_lo, c->fb, c->fb_range,
                            clips, p.R0, 1, p.F_max, mel, s);
    }));
  } else {
    GAM_TRY(upload_table(c, p, s, &clips));
    GAM_TRY(run_kernel(c, PK_FRONTEND, s, [&] {
      return launch_frontend(audio, max_samples, clips, batch * p.F_max, 0, p.F_max, c->basis, c->fb, mel, 0, s);
    }));
  }
  if (frames_out)
    for (int i = 0; i < batch; ++i) frames_out[i] = p.len[i].F;
  return GAM_OK;
}

gam_status gam_encode(gam_ctx* c, const float* audio, const int32_t* lengths, int batch, int64_t max_samples,
                      float* enc, int32_t* enc_len_out, void* stream) {
  GAM_TRY(enter(c));
  return run_encoder(c, audio, lengths, batch, max_samples, -1, -1, enc, enc_len_out, (cudaStream_t)stream);
}

gam_status gam_encode_stage(gam_ctx* c, const float* audio, const int32_t* lengths, int batch, int64_t max_samples,
                            int layer, int stage, float* out, void* stream) {
  GAM_TRY(enter(c));
  if (stage < GAM_STAGE_SUBSAMPLING || stage > GAM_STAGE_LAYER) return fail(c, GAM_ERR_INVALID_ARG, "bad stage");
  if (stage != GAM_STAGE_SUBSAMPLING && (layer < 0 || layer >= c->cfg.n_layers))
    return fail(c, GAM_ERR_INVALID_ARG, "layer out of range");
  return run_encoder(c, audio, lengths, batch, max_samples, layer, stage, out, nullptr, (cudaStream_t)stream);
}

gam_status gam_ctc_greedy(gam_ctx* c, const float* enc, const int32_t* enc_len, int batch, int t_max, float* logp,
                          int32_t* tokens, int32_t* counts, void* stream) {
  GAM_TRY(enter(c));
  return run_ctc(c, enc, enc_len, batch, t_max, logp, tokens, counts, (cudaStream_t)stream);
}

gam_status gam_ctc_greedy_frames(gam_ctx* c, const float* enc, const int32_t* enc_len, int batch, int t_max,
                                 int32_t* tokens, int32_t* frames, int32_t* counts, void* stream) {
  GAM_TRY(enter(c));
  if (!frames) return fail(c, GAM_ERR_INVALID_ARG, "null frames pointer");
  return run_ctc(c, enc, enc_len, batch, t_max, nullptr, tokens, counts, (cudaStream_t)stream, frames);
}

gam_status gam_ctc_collapse(gam_ctx* c, const float* logits, const int32_t* lengths, int batch, int t_max,
                            int n_classes, int32_t* tokens, int32_t* counts, void* stream) {
  GAM_TRY(enter(c));
  if (!logits || !lengths || !tokens || !counts) return fail(c, GAM_ERR_INVALID_ARG, "null pointer");
  if (batch < 1 || t_max < 1 || n_classes < 2) return fail(c, GAM_ERR_INVALID_ARG, "bad sizes");
  if ((int64_t)batch * t_max > (int64_t)c->cfg.max_batch * c->T2_cap)
    return fail(c, GAM_ERR_CAPACITY, "batch * t_max above the context's capacity");
  for (int i = 0; i < batch; ++i)
    if (lengths[i] < 0 || lengths[i] > t_max) return fail(c, GAM_ERR_SHAPE, "length outside [0, t_max]");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  const int* lens;
  GAM_TRY(upload_ints(c, lengths, batch, s, &lens));
  GAM_TRY(run_kernel(c, PK_CTC_SOFTMAX, s, [&] {
    return launch_logsoftmax_argmax(logits, n_classes, lens, batch, t_max, n_classes, nullptr, c->argmax, s);
  }));
  return run_kernel(c, PK_CTC_COLLAPSE, s, [&] {
    return launch_collapse(c->argmax, lens, batch, t_max, n_classes - 1, tokens, counts, s);
  });
}

gam_status gam_transcribe(gam_ctx* c, const float* audio_host, const int32_t* lengths, int batch, int64_t max_samples,
                          int32_t* tokens_host, int32_t* counts_host, void* stream) {
  GAM_TRY(enter(c));
  if (!audio_host || !tokens_host || !counts_host) return fail(c, GAM_ERR_INVALID_ARG, "null pointer");
  if (batch > c->cfg.max_batch || max_samples > c->cfg.max_samples)
    return fail(c, GAM_ERR_CAPACITY, "batch or max_samples above capacity");
  Plan p;
  GAM_TRY(make_plan(c, c->cfg, lengths, batch, max_samples, p));
  cudaStream_t s = (cudaStream_t)stream;
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(c->audio_stage, audio_host, (size_t)batch * max_samples * 4,
                                        cudaMemcpyHostToDevice, s), "audio upload"));
  std::vector<int32_t> enc_len(batch);
  GAM_TRY(run_encoder(c, c->audio_stage, lengths, batch, max_samples, -1, -1, c->enc_stage, enc_len.data(), s));
  GAM_TRY(run_ctc(c, c->enc_stage, enc_len.data(), batch, p.T2_max, nullptr, c->tokens_stage, c->counts_stage, s));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(tokens_host, c->tokens_stage, (size_t)batch * p.T2_max * 4,
                                        cudaMemcpyDeviceToHost, s), "tokens download"));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(counts_host, c->counts_stage, (size_t)batch * 4, cudaMemcpyDeviceToHost, s),
                     "counts download"));
  return cuda_check(c, cudaStreamSynchronize(s), "transcribe sync");
}

gam_status gam_graphs_enable(gam_ctx* c, int on) {
  GAM_TRY(enter(c));
  c->graphs.enabled = on != 0;
  c->graphs.seen.clear();
  return GAM_OK;
}

gam_status gam_device_status(gam_ctx* c) {
  GAM_TRY(enter(c));
  GAM_TRY(cuda_check(c, cudaStreamSynchronize(c->last_stream), "stream sync"));
  int st[4] = {0, 0, 0, 0};
  GAM_TRY(cuda_check(c, cudaMemcpy(st, c->dev_status, 16, cudaMemcpyDeviceToHost), "status read"));
  int tc_st = 0;
  GAM_TRY(cuda_check(c, tc_read_status(&c->tc, &tc_st), "status read"));
  if (st[0] != 0 || tc_st != 0) return fail(c, GAM_ERR_DEVICE_TIMEOUT, "a device-side wait gave up");
  return GAM_OK;
}

gam_status gam_profile_enable(gam_ctx* c, int on) {
  GAM_TRY(enter(c));
  GAM_TRY(gam_profile_reset(c));
  c->prof.mask = (uint32_t)on & ((1u << PK_COUNT) - 1u);
  return GAM_OK;
}

gam_status gam_profile_reset(gam_ctx* c) {
  GAM_TRY(enter(c));
  GAM_TRY(cuda_check(c, cudaDeviceSynchronize(), "profile sync"));
  for (int k = 0; k < PK_COUNT; ++k) {
    c->prof.launches[k] = 0;
    c->prof.ms[k] = 0.0;
  }
  c->prof.npairs = 0;
  GAM_TRY(cuda_check(c, cudaMemset(c->dev_status, 0, 16), "status reset"));
  return cuda_check(c, tc_reset_status(&c->tc), "status reset");
}

int gam_profile_kinds(void) { return PK_COUNT; }

const char* gam_profile_kind_name(int kind) { return (kind >= 0 && kind < PK_COUNT) ? kKindNames[kind] : ""; }

gam_status gam_profile_read(gam_ctx* c, int kind, double* total_ms, int64_t* launches) {
  GAM_TRY(enter(c));
  if (kind < 0 || kind >= PK_COUNT) return fail(c, GAM_ERR_INVALID_ARG, "bad kind");
  Prof& p = c->prof;
  if (p.npairs > 0) {
    GAM_TRY(cuda_check(c, cudaEventSynchronize(p.ev[2 * p.npairs - 1]), "profile sync"));
    for (int i = 0; i < p.npairs; ++i) {
      if (p.pair_kind[i] < 0) continue;
      float t = 0.f;
      GAM_TRY(cuda_check(c, cudaEventElapsedTime(&t, p.ev[2 * i], p.ev[2 * i + 1]), "event time"));
      p.ms[p.pair_kind[i]] += (double)t;
    }
    p.npairs = 0;
  }
  if (total_ms) *total_ms = p.ms[kind];
  if (launches) *launches = p.launches[kind];
  return GAM_OK;
}

gam_status gam_debug_gemm(gam_ctx* c, int impl, const void* a, int lda, const void* w, const float* bias, int m, int n,
                          int k, float* out, int ldo, void* stream) {
  GAM_TRY(enter(c));
  if (!a || !w || !bias || !out || m < 1 || n < 1 || k < 1 || lda < 1 || ldo < n)
    return fail(c, GAM_ERR_INVALID_ARG, "bad gemm arguments");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  EpiParams ep{};
  ep.x = out;
  ep.out = out;
  ep.bias = bias;
  ep.alpha = 1.f;
  ep.ldo = ldo;
  WeightOp W{w, nullptr, 1, nullptr};
  const int kind = impl & 0xff, width = impl >> 8;
  if (impl < 0 || kind > 4 || ((kind == 1 || kind == 4) && width) ||
      (width && width != 64 && width != 128 && width != 192 && width != 256) || (width == 64 && kind == 3))
    return fail(c, GAM_ERR_INVALID_ARG, "impl: kind 0 .. 4 plus (tile width 64 (single-CTA), 128, 192 or 256) << 8");
  if (kind != 1) {
    if (!tc_supported(1, 1, n, k, EPI_RESID)) return fail(c, GAM_ERR_SHAPE, "tensor-core GEMM needs N % 256 == 0, K % 64 == 0");
    const int variant = kind == 0 ? -1 : kind == 2 ? 0 : kind == 3 ? 1 : 2;
    if (kind == 4 && (m > 256 || lda < k))
      return fail(c, GAM_ERR_SHAPE, "split-K GEMM: at most 256 rows, plain A operand");
    if (kind != 4 && !choose_tile(&c->tc, m, n, EPI_RESID, false, variant, width).width)
      return fail(c, GAM_ERR_SHAPE, "no tile of that width divides N");
    return run_kernel(c, PK_MISC, s, [&] {
      return launch_gemm_tc(&c->tc, a, nullptr, 0, lda, W, m, n, k, EPI_RESID, ep, s, variant, width);
    });
  }
  if (k % 16 || n % 128) return fail(c, GAM_ERR_SHAPE, "CUDA-core GEMM needs N % 128 == 0, K % 16 == 0");
  return run_kernel(c, PK_MISC, s, [&] { return launch_gemm_simt(1, a, nullptr, 0, lda, W, m, n, k, EPI_RESID, 0, ep, s); });
}

gam_status gam_rnnt_attach(gam_ctx* c, const gam_rnnt_config* cfg, const gam_tensor* tensors, int n_tensors) {
  GAM_TRY(enter(c));
  if (!cfg || !tensors || n_tensors <= 0) return fail(c, GAM_ERR_INVALID_ARG, "null config or no tensors");
  return rnnt_attach(c, *cfg, tensors, n_tensors);
}

gam_status gam_rnnt_greedy(gam_ctx* c, const float* enc, const int32_t* enc_len, int batch, int t_max,
                           int max_tokens, int32_t* tokens, int32_t* frames, int32_t* counts, void* stream) {
  GAM_TRY(enter(c));
  return rnnt_greedy(c, enc, enc_len, batch, t_max, max_tokens, tokens, frames, counts, (cudaStream_t)stream);
}

gam_status gam_stream_create(gam_ctx* c, int64_t window_samples, gam_stream** out) {
  GAM_TRY(enter(c));
  if (!out) return fail(c, GAM_ERR_INVALID_ARG, "null output pointer");
  *out = nullptr;
  if (window_samples < 1280 || window_samples > c->cfg.max_samples)
    return fail(c, GAM_ERR_CAPACITY, "window must be 1280 samples .. the context's max_samples");
  gam_stream* st = new gam_stream();
  st->ctx = c;
  st->window = window_samples;
  ClipLen l = clip_len(window_samples, c->cfg);
  st->t_cap = l.T2;
  auto alloc = [&](void** p, size_t bytes) {
    cudaError_t e = cudaMalloc(p, bytes);
    if (e == cudaSuccess) st->allocs.push_back(*p);
    return cuda_check(c, e, "cudaMalloc");
  };
  gam_status s = alloc((void**)&st->buf[0], (size_t)window_samples * 4);
  if (s == GAM_OK) s = alloc((void**)&st->buf[1], (size_t)window_samples * 4);
  if (s == GAM_OK) s = alloc((void**)&st->enc, (size_t)st->t_cap * c->cfg.d_model * 4);
  if (s == GAM_OK) s = alloc((void**)&st->tok, (size_t)st->t_cap * 4);
  if (s == GAM_OK) s = alloc((void**)&st->cnt, 16);
  if (s == GAM_OK)
    s = cuda_check(c, cudaMallocHost((void**)&st->tok_host, ((size_t)st->t_cap + 1) * 4), "cudaMallocHost");
  if (s != GAM_OK) {
    gam_stream_destroy(st);
    return s;
  }
  *out = st;
  return GAM_OK;
}

gam_status gam_stream_destroy(gam_stream* st) {
  if (!st) return GAM_OK;
  if (st->ctx) cudaSetDevice(st->ctx->device);
  cudaDeviceSynchronize();
  for (void* p : st->allocs) cudaFree(p);
  if (st->tok_host) cudaFreeHost(st->tok_host);
  delete st;
  return GAM_OK;
}

gam_status gam_stream_reset(gam_stream* st) {
  if (!st) return GAM_ERR_INVALID_ARG;
  st->len = 0;
  st->total = 0;
  return GAM_OK;
}

gam_status gam_stream_push(gam_stream* st, const float* samples_host, int64_t n, int32_t* tokens_host,
                           int max_tokens, int32_t* count_out, int64_t* window_start_out, void* stream) {
  if (!st) return GAM_ERR_INVALID_ARG;
  gam_ctx* c = st->ctx;
  GAM_TRY(enter(c));
  if (n < 0 || (n > 0 && !samples_host) || !tokens_host || !count_out || max_tokens < 0)
    return fail(c, GAM_ERR_INVALID_ARG, "bad push arguments");
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  // new window = the last `window` samples of (old window + new samples), written to the other buffer
  const int64_t keep_new = std::min(n, st->window);
  const int64_t keep_old = std::min(st->len, st->window - keep_new);
  float* dst = st->buf[st->cur ^ 1];
  if (keep_old > 0)
    GAM_TRY(cuda_check(c, cudaMemcpyAsync(dst, st->buf[st->cur] + (st->len - keep_old), (size_t)keep_old * 4,
                                          cudaMemcpyDeviceToDevice, s), "window copy"));
  if (keep_new > 0)
    GAM_TRY(cuda_check(c, cudaMemcpyAsync(dst + keep_old, samples_host + (n - keep_new), (size_t)keep_new * 4,
                                          cudaMemcpyHostToDevice, s), "samples upload"));
  st->cur ^= 1;
  st->len = keep_old + keep_new;
  st->total += n;
  if (window_start_out) *window_start_out = st->total - st->len;
  *count_out = 0;
  if (st->len < 1280) return cuda_check(c, cudaStreamSynchronize(s), "stream sync");  // no encoder frame yet
  const int32_t len32 = (int32_t)st->len;
  int32_t el = 0;
  GAM_TRY(run_encoder(c, st->buf[st->cur], &len32, 1, st->len, -1, -1, st->enc, &el, s));
  GAM_TRY(run_ctc(c, st->enc, &el, 1, el, nullptr, st->tok, st->cnt, s));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(st->tok_host, st->cnt, 4, cudaMemcpyDeviceToHost, s), "count download"));
  GAM_TRY(cuda_check(c, cudaMemcpyAsync(st->tok_host + 1, st->tok, (size_t)el * 4, cudaMemcpyDeviceToHost, s),
                     "tokens download"));
  GAM_TRY(cuda_check(c, cudaStreamSynchronize(s), "stream sync"));
  const int cnt = st->tok_host[0];
  *count_out = cnt;
  std::memcpy(tokens_host, st->tok_host + 1, (size_t)std::min(cnt, max_tokens) * 4);
  return GAM_OK;
}

gam_status gam_debug_wait_timeout(gam_ctx* c, int64_t limit_ns, int skip_k_block) {
  GAM_TRY(enter(c));
  if (limit_ns <= 0) return fail(c, GAM_ERR_INVALID_ARG, "limit_ns must be positive");
  c->tc.debug_limit_ns = (uint64_t)limit_ns;
  c->tc.debug_skip = skip_k_block >= 0 ? skip_k_block : -1;
  return GAM_OK;
}

gam_status gam_debug_inject_cuda_error(gam_ctx* c, int cuda_error, int count) {
  if (!c) return GAM_ERR_INVALID_ARG;
  c->inject_err = cuda_error;
  c->inject_count = count;
  return GAM_OK;
}

}  // extern "C"
