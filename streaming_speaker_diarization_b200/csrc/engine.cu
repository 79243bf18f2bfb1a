// Host side of libsf.so: the C ABI declared in include/sf.h.
//
// One engine = one set of weights on one device.  Weights are converted once
// (bf16 or fp32), BatchNorm is folded into the depthwise conv, the GLU
// projection is interleaved so each (value, gate) pair lands in one thread of
// the GEMM epilogue, Q/K/V are concatenated into one projection, the
// subsampling Linear's columns are permuted to the channels-last flattening,
// and every conformer layer's relative-position projection pe . W_pos^T is
// precomputed for all distances |i - j| < R (it depends on weights only).
//
// Every call is described to the kernels by one descriptor block (sequence
// offsets, window positions, per-stream sizes) copied host -> device at the
// start of the call; sizes of the streaming state are data-independent and
// tracked on the host, contents stay on the device.
#include <cuda_runtime.h>
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <algorithm>
#include <memory>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/sf.h"
#include "blob.h"
#include "common.cuh"
#include "frontend.h"
#include "layers.h"
#include "stream.h"

using namespace sf;

// Per-call context is per host thread, so that engines driven from
// different threads (e.g. one per GPU) do not see each other's calls.
namespace sf {
thread_local int g_launch_pdl = 0;
}

// Source line of the first CUDA call that failed in the current API call
// (reported by sf_last_error).
static thread_local int g_fail_line = 0;
#define CK(x)                                   \
  do {                                          \
    cudaError_t _e = (x);                       \
    if (_e != cudaSuccess) {                    \
      if (!g_fail_line) g_fail_line = __LINE__; \
      return _e;                                \
    }                                           \
  } while (0)

namespace {

struct Buf {
  void* p = nullptr;
  size_t bytes = 0;
};

struct DescBlock {
  SeqTable seq;
  int64_t len[MAX_SEQ];
  int buf[MAX_SEQ];
  int64_t start[MAX_SEQ];
  int64_t frames[MAX_SEQ];
  int first[MAX_SEQ];
  int count[MAX_SEQ];
  int dst[MAX_SEQ];
  int n_cand[MAX_SEQ];
  int64_t win_f0[MAX_SEQ];   // audio-in steps: first mel frame of each window
  int64_t win_a0[MAX_SEQ];   //   absolute sample of the stream's buffer column 0
  int win_nf[MAX_SEQ];       //   mel frames of the window
  StepDesc step;
};

template <typename T> struct ConfW {
  float *ff1_g, *ff1_b, *ff1_b1, *ff1_b2;
  T *ff1_w1, *ff1_w2;
  float *att_g, *att_b, *bqkv, *bo, *pu, *pv;
  T *wqkv, *wo;
  T* ptab;   // [(2R-1) x 512], rows r = -(R-1) .. R-1
  float *conv_g, *conv_b, *pw1_b, *dw_w, *dw_b, *pw2_b;
  T *pw1, *pw2;
  float *ff2_g, *ff2_b, *ff2_b1, *ff2_b2;
  T *ff2_w1, *ff2_w2;
  float *out_g, *out_b;
};
template <typename T> struct TfW {
  T *wqkv, *wo, *w1, *w2;
  float *bqkv, *bo, *ln1_g, *ln1_b, *b1, *b2, *ln2_g, *ln2_b;
};
template <typename T> struct Weights {
  float *c1_w, *c1_b, *dw_w[2], *dw_b[2], *pw_b[2], *out_b;
  T *pw_w[2], *out_w;
  std::vector<ConfW<T>> conf;
  T* proj_w;
  float* proj_b;
  std::vector<TfW<T>> tf;
  T* head_w1;
  float *head_b1, *head_w2, *head_b2;
};

// Host staging arena: tensors appended 256-byte aligned, uploaded once, then
// the recorded pointer slots are patched to device addresses.
struct Arena {
  std::vector<uint8_t> host;
  std::vector<std::pair<void**, size_t>> fix;
  template <typename P> void add(P** slot, const void* src, size_t bytes) {
    size_t off = (host.size() + 255) & ~size_t(255);
    host.resize(off + bytes);
    memcpy(host.data() + off, src, bytes);
    fix.push_back({reinterpret_cast<void**>(slot), off});
  }
};

}  // namespace

namespace {
constexpr size_t SPLIT_WS_BYTES = (size_t)40 << 20;
constexpr int SPLIT_CNT = 1 << 16;
enum KClass : int {
  K_MEL = 0, K_CONV1, K_DW2D, K_GEMM, K_ATT_REL, K_ATT_MHA, K_LN, K_DW1D, K_HEAD, K_ASSEMBLE, K_EXTRACT,
  K_UPDATE, K_TOF32, K_SELECT, K_TFL, K_COUNT
};
const char* const KNAMES[K_COUNT] = {"mel", "conv1", "dwconv3x3s2", "gemm", "attention_relpos", "attention_mha",
                                     "layernorm", "dwconv1d", "head_out", "assemble", "extract", "state_update",
                                     "to_f32", "select_topk", "tf_layer"};
struct ProfRec {
  int cls;
  cudaEvent_t a, b;
};
}  // namespace

struct sf_engine {
  sf_config cfg{};
  int device = 0;
  int n_sms = 148;        // streaming multiprocessors of the device
  std::string err;
  int R = 0;              // position-table half length (longest sequence)
  int max_seq_len = 0;
  void* d_weights = nullptr;
  void* d_ptab = nullptr;
  MelTables* d_mel_tab = nullptr;
  DescBlock* h_desc = nullptr;
  DescBlock* d_desc = nullptr;
  cudaEvent_t desc_ev = nullptr;
  bool desc_pending = false;
  int* d_err = nullptr;
  int gemm_path = 1;      // bf16 GEMMs: tcgen05 with CTA pairs 1 = where faster (default), 2 = always,
                          // 3 = never; 0 = mma.sync
  int pair_bn = 0;        // CTA-pair tile width (0 = planned)
  int attn_path = 1;      // bf16 relative-position attention: 1 = tcgen05, 0 = mma.sync
  int mel_path = MEL_DEFAULT_PATH;   // front-end: 1 = register FFT + all-SM normalisation, 0 = shared-memory FFT
  int sub_path = 1;       // subsampling: 1 = conv1 fused into the first depthwise, 0 = conv1 and depthwise kernels
  int ln_fuse = 1;        // bf16: LayerNorm fused into the residual projections' epilogue where it fits
  int tf_fuse = 1;        // bf16 Transformer layers after the attention: 1 fused where one wave covers the rows,
                          // 2 fused always, 0 separate projections and LayerNorms
  float* d_split_ws = nullptr;   // split-K partial tiles of the tcgen05 GEMM
  int* d_split_cnt = nullptr;    // their per-tile arrival counters (kept at zero between launches)
  TcScratch tc_scratch() const { return TcScratch{d_err, d_split_ws, SPLIT_WS_BYTES, d_split_cnt, SPLIT_CNT}; }
  Weights<float> wf;
  Weights<bf16> wb;
  // profiling: launch/work counters always; event pairs when prof is set
  bool prof = false;
  uint32_t prof_mask = 0;       // kernel classes bracketed with events
  int64_t launches[K_COUNT] = {};
  double kflops[K_COUNT] = {};
  double kbytes[K_COUNT] = {};
  std::vector<ProfRec> recs;
  std::vector<cudaEvent_t> pool;
  size_t pool_used = 0;
  double att_s2 = 0;      // sum of squared sequence lengths of the current call
  int att_tiles2 = 0;     // 128-row attention query tiles of the current call
  int att_max_len = 0;    // longest sequence of the current call
  double ms_acc[K_COUNT] = {};   // event time already read back (graph replays)
  // CUDA graphs: one per launch shape, replayed; invalidated when the workspace moves
  bool use_graphs = true;
  int use_pdl = 1;         // programmatic dependent launch (measured 4.5 % faster offline; bitwise equal)
  bool capturing = false;
  cudaStream_t cap_stream = nullptr;     // graphs are captured here, launched on the caller's stream
  std::vector<cudaEvent_t> cap_events;   // events created for the graph being captured
  uint64_t ws_gen = 0;
  struct GraphEntry {
    cudaGraphExec_t exec = nullptr;
    uint64_t gen = 0;
    int64_t launches[K_COUNT] = {};
    double flops[K_COUNT] = {}, bytes[K_COUNT] = {};
    std::vector<ProfRec> recs;
    std::vector<cudaEvent_t> events;
  };
  std::unordered_map<std::string, GraphEntry> graphs;
  uint64_t stream_serial = 0;   // last serial handed to a stream
  std::vector<sf_stream*> streams;   // live streams (detached when the engine goes first)
  // workspace (grow-only)
  Buf mel, part, audio, sub1, sub2a, sub2b, sub3a, sub3b, emb, x, h, big, ctx, x2, h2, probs, out;
};

struct sf_stream {
  sf_engine* e = nullptr;
  uint64_t serial = 0;    // identifies the stream's graphs (a host address may be reused after destroy)
  sf_preset p{};
  int n = 0;
  StateBufs sb{};
  void* alloc = nullptr;
  std::vector<int> n_c, n_f, cur_c, cur_f, finished;
  std::vector<int64_t> c0;
};

namespace {

sf_status fail(sf_engine* e, sf_status s, const std::string& msg) {
  if (e) e->err = msg;
  return s;
}
sf_status cuda_fail(sf_engine* e, cudaError_t c, const char* where) {
  std::string msg = std::string(where) + ": " + cudaGetErrorString(c);
  if (g_fail_line) msg += " (engine.cu:" + std::to_string(g_fail_line) + ")";
  g_fail_line = 0;
  return fail(e, c == cudaErrorMemoryAllocation ? SF_ENOMEM : SF_ECUDA, msg);
}

cudaEvent_t pool_event(sf_engine* e) {
  if (e->pool_used == e->pool.size()) {
    cudaEvent_t ev;
    if (cudaEventCreate(&ev) != cudaSuccess) return nullptr;
    e->pool.push_back(ev);
  }
  return e->pool[e->pool_used++];
}

cudaEvent_t cap_event(sf_engine* e) {
  cudaEvent_t ev;
  if (cudaEventCreate(&ev) != cudaSuccess) return nullptr;
  e->cap_events.push_back(ev);
  return ev;
}

// Accounts one launch site: counters always, an event pair when profiling.
struct Scope {
  sf_engine* e;
  cudaStream_t st;
  cudaEvent_t b = nullptr;
  Scope(sf_engine* e_, int cls, int n_kernels, double flops, double bytes, cudaStream_t st_) : e(e_), st(st_) {
    e->launches[cls] += n_kernels;
    e->kflops[cls] += flops;
    e->kbytes[cls] += bytes;
    if (e->prof && ((e->prof_mask >> cls) & 1u)) {
      cudaEvent_t a = e->capturing ? cap_event(e) : pool_event(e);
      b = e->capturing ? cap_event(e) : pool_event(e);
      if (a && b) {
        // inside a capture, only an "external" record becomes an event node of the graph
        cudaEventRecordWithFlags(a, st, e->capturing ? cudaEventRecordExternal : cudaEventRecordDefault);
        e->recs.push_back({cls, a, b});
      } else {
        b = nullptr;
      }
    }
  }
  ~Scope() {
    if (b) cudaEventRecordWithFlags(b, st, e->capturing ? cudaEventRecordExternal : cudaEventRecordDefault);
  }
};
#define RUN(cls, nk, flops, bytes, call)                 \
  do {                                                   \
    Scope _scope(e, cls, nk, (double)(flops), (double)(bytes), st); \
    CK(call);                                            \
  } while (0)

thread_local uint64_t* g_ws_gen = nullptr;   // generation counter of the engine whose buffers ensure() grows

cudaError_t ensure(Buf& b, size_t bytes) {
  if (bytes <= b.bytes) return cudaSuccess;
  if (g_ws_gen) ++*g_ws_gen;
  if (b.p) CK(cudaFree(b.p));
  b.p = nullptr;
  b.bytes = 0;
  bytes = (bytes + 4095) & ~size_t(4095);
  CK(cudaMalloc(&b.p, bytes));
  b.bytes = bytes;
  return cudaSuccess;
}

size_t act_size(const sf_engine* e) { return e->cfg.precision == SF_BF16 ? 2 : 4; }

inline int64_t enc_frames(int64_t L) { return L <= 0 ? 0 : 1 + (L - 1) / 8; }
inline int64_t half_len(int64_t l) { return 1 + (l - 1) / 2; }

template <typename T> void to_act(const std::vector<float>& src, std::vector<uint8_t>& dst) {
  dst.resize(src.size() * sizeof(T));
  if (sizeof(T) == 4) {
    memcpy(dst.data(), src.data(), src.size() * 4);
  } else {
    uint16_t* d = reinterpret_cast<uint16_t*>(dst.data());
    for (size_t i = 0; i < src.size(); ++i) d[i] = f2bf_bits(src[i]);
  }
}

template <typename T> struct Builder {
  Arena& a;
  void f32(float** slot, const float* src, size_t n) { a.add(slot, src, n * 4); }
  void f32v(float** slot, const std::vector<float>& v) { a.add(slot, v.data(), v.size() * 4); }
  void act(T** slot, const std::vector<float>& v) {
    std::vector<uint8_t> tmp;
    to_act<T>(v, tmp);
    a.add(slot, tmp.data(), tmp.size());
  }
  void actp(T** slot, const float* src, size_t n) { act(slot, std::vector<float>(src, src + n)); }
};

std::vector<float> vec(const float* p, size_t n) { return std::vector<float>(p, p + n); }

template <typename T>
sf_status load_weights(sf_engine* e, std::unordered_map<std::string, TensorRef>& m, Weights<T>& W) {
  const sf_config& c = e->cfg;
  const int D = c.d_model, E = c.tf_d_model, C = 256, F3 = c.n_mels / 8, DFF = D * c.ff_mult, K = c.conv_kernel;
  Loader L{m, ""};
  Arena arena;
  Builder<T> B{arena};
  const std::string pre = "enc.pre_encode.";
  const float* p;
  if ((p = L.get(pre + "conv1.weight", {(uint32_t)C, 1, 3, 3}))) B.f32(&W.c1_w, p, C * 9);
  if ((p = L.get(pre + "conv1.bias", {(uint32_t)C}))) B.f32(&W.c1_b, p, C);
  for (int s = 0; s < 2; ++s) {
    const std::string t = std::to_string(s + 1);
    if ((p = L.get(pre + "dw" + t + ".weight", {(uint32_t)C, 1, 3, 3}))) B.f32(&W.dw_w[s], p, C * 9);
    if ((p = L.get(pre + "dw" + t + ".bias", {(uint32_t)C}))) B.f32(&W.dw_b[s], p, C);
    if ((p = L.get(pre + "pw" + t + ".weight", {(uint32_t)C, (uint32_t)C}))) B.actp(&W.pw_w[s], p, C * C);
    if ((p = L.get(pre + "pw" + t + ".bias", {(uint32_t)C}))) B.f32(&W.pw_b[s], p, C);
  }
  if ((p = L.get(pre + "out.weight", {(uint32_t)D, (uint32_t)(C * F3)}))) {
    // torch flattening is c * F3 + f; the engine's rows are f * C + c
    std::vector<float> w((size_t)D * C * F3);
    for (int n = 0; n < D; ++n)
      for (int ch = 0; ch < C; ++ch)
        for (int f = 0; f < F3; ++f) w[(size_t)n * C * F3 + f * C + ch] = p[(size_t)n * C * F3 + ch * F3 + f];
    B.act(&W.out_w, w);
  }
  if ((p = L.get(pre + "out.bias", {(uint32_t)D}))) B.f32(&W.out_b, p, D);

  W.conf.resize(c.n_conformer);
  for (int l = 0; l < c.n_conformer; ++l) {
    ConfW<T>& w = W.conf[l];
    const std::string q = "enc.layers." + std::to_string(l) + ".";
    auto ffn = [&](const std::string& tag, float** g, float** b, T** w1, float** b1, T** w2, float** b2) {
      if ((p = L.get(q + tag + ".ln.weight", {(uint32_t)D}))) B.f32(g, p, D);
      if ((p = L.get(q + tag + ".ln.bias", {(uint32_t)D}))) B.f32(b, p, D);
      if ((p = L.get(q + tag + ".linear1.weight", {(uint32_t)DFF, (uint32_t)D}))) B.actp(w1, p, (size_t)DFF * D);
      if ((p = L.get(q + tag + ".linear1.bias", {(uint32_t)DFF}))) B.f32(b1, p, DFF);
      if ((p = L.get(q + tag + ".linear2.weight", {(uint32_t)D, (uint32_t)DFF}))) B.actp(w2, p, (size_t)DFF * D);
      if ((p = L.get(q + tag + ".linear2.bias", {(uint32_t)D}))) B.f32(b2, p, D);
    };
    ffn("ff1", &w.ff1_g, &w.ff1_b, &w.ff1_w1, &w.ff1_b1, &w.ff1_w2, &w.ff1_b2);
    if ((p = L.get(q + "att.ln.weight", {(uint32_t)D}))) B.f32(&w.att_g, p, D);
    if ((p = L.get(q + "att.ln.bias", {(uint32_t)D}))) B.f32(&w.att_b, p, D);
    {
      std::vector<float> wq, bq;
      for (const char* nm : {"q", "k", "v"}) {
        const float* pw = L.get(q + "att.linear_" + nm + ".weight", {(uint32_t)D, (uint32_t)D});
        const float* pb = L.get(q + "att.linear_" + nm + ".bias", {(uint32_t)D});
        if (!pw || !pb) break;
        wq.insert(wq.end(), pw, pw + (size_t)D * D);
        bq.insert(bq.end(), pb, pb + D);
      }
      if (wq.size() == (size_t)3 * D * D) {
        B.act(&w.wqkv, wq);
        B.f32v(&w.bqkv, bq);
      }
    }
    if ((p = L.get(q + "att.linear_out.weight", {(uint32_t)D, (uint32_t)D}))) B.actp(&w.wo, p, (size_t)D * D);
    if ((p = L.get(q + "att.linear_out.bias", {(uint32_t)D}))) B.f32(&w.bo, p, D);
    L.get(q + "att.linear_pos.weight", {(uint32_t)D, (uint32_t)D});
    const int H = c.n_heads, dk = D / H;
    if ((p = L.get(q + "att.pos_bias_u", {(uint32_t)H, (uint32_t)dk}))) B.f32(&w.pu, p, D);
    if ((p = L.get(q + "att.pos_bias_v", {(uint32_t)H, (uint32_t)dk}))) B.f32(&w.pv, p, D);
    if ((p = L.get(q + "conv.ln.weight", {(uint32_t)D}))) B.f32(&w.conv_g, p, D);
    if ((p = L.get(q + "conv.ln.bias", {(uint32_t)D}))) B.f32(&w.conv_b, p, D);
    {
      const float* pw = L.get(q + "conv.pointwise1.weight", {(uint32_t)(2 * D), (uint32_t)D});
      const float* pb = L.get(q + "conv.pointwise1.bias", {(uint32_t)(2 * D)});
      if (pw && pb) {   // interleave (value_c, gate_c) rows for the GLU epilogue
        std::vector<float> wi((size_t)2 * D * D), bi(2 * D);
        for (int ch = 0; ch < D; ++ch) {
          memcpy(&wi[(size_t)(2 * ch) * D], pw + (size_t)ch * D, D * 4);
          memcpy(&wi[(size_t)(2 * ch + 1) * D], pw + (size_t)(D + ch) * D, D * 4);
          bi[2 * ch] = pb[ch];
          bi[2 * ch + 1] = pb[D + ch];
        }
        B.act(&w.pw1, wi);
        B.f32v(&w.pw1_b, bi);
      }
    }
    {
      const float* dw = L.get(q + "conv.depthwise.weight", {(uint32_t)D, (uint32_t)K});
      const float* db = L.get(q + "conv.depthwise.bias", {(uint32_t)D});
      const float* mu = L.get(q + "conv.bn.running_mean", {(uint32_t)D});
      const float* var = L.get(q + "conv.bn.running_var", {(uint32_t)D});
      const float* ga = L.get(q + "conv.bn.weight", {(uint32_t)D});
      const float* be = L.get(q + "conv.bn.bias", {(uint32_t)D});
      if (dw && db && mu && var && ga && be) {   // fold BatchNorm (running statistics)
        std::vector<float> fw((size_t)D * K), fb(D);
        for (int ch = 0; ch < D; ++ch) {
          const double sc = (double)ga[ch] / sqrt((double)var[ch] + 1e-5);
          for (int j = 0; j < K; ++j) fw[(size_t)ch * K + j] = (float)(dw[(size_t)ch * K + j] * sc);
          fb[ch] = (float)(((double)db[ch] - mu[ch]) * sc + be[ch]);
        }
        B.f32v(&w.dw_w, fw);
        B.f32v(&w.dw_b, fb);
      }
    }
    if ((p = L.get(q + "conv.pointwise2.weight", {(uint32_t)D, (uint32_t)D}))) B.actp(&w.pw2, p, (size_t)D * D);
    if ((p = L.get(q + "conv.pointwise2.bias", {(uint32_t)D}))) B.f32(&w.pw2_b, p, D);
    ffn("ff2", &w.ff2_g, &w.ff2_b, &w.ff2_w1, &w.ff2_b1, &w.ff2_w2, &w.ff2_b2);
    if ((p = L.get(q + "out_ln.weight", {(uint32_t)D}))) B.f32(&w.out_g, p, D);
    if ((p = L.get(q + "out_ln.bias", {(uint32_t)D}))) B.f32(&w.out_b, p, D);
  }
  if ((p = L.get("proj.weight", {(uint32_t)E, (uint32_t)D}))) B.actp(&W.proj_w, p, (size_t)E * D);
  if ((p = L.get("proj.bias", {(uint32_t)E}))) B.f32(&W.proj_b, p, E);
  W.tf.resize(c.n_transformer);
  for (int l = 0; l < c.n_transformer; ++l) {
    TfW<T>& w = W.tf[l];
    const std::string q = "tf.layers." + std::to_string(l) + ".";
    std::vector<float> wq, bq;
    for (const char* nm : {"q", "k", "v"}) {
      const float* pw = L.get(q + "att." + nm + ".weight", {(uint32_t)E, (uint32_t)E});
      const float* pb = L.get(q + "att." + nm + ".bias", {(uint32_t)E});
      if (!pw || !pb) break;
      wq.insert(wq.end(), pw, pw + (size_t)E * E);
      bq.insert(bq.end(), pb, pb + E);
    }
    if (wq.size() == (size_t)3 * E * E) {
      B.act(&w.wqkv, wq);
      B.f32v(&w.bqkv, bq);
    }
    if ((p = L.get(q + "att.o.weight", {(uint32_t)E, (uint32_t)E}))) B.actp(&w.wo, p, (size_t)E * E);
    if ((p = L.get(q + "att.o.bias", {(uint32_t)E}))) B.f32(&w.bo, p, E);
    if ((p = L.get(q + "ln1.weight", {(uint32_t)E}))) B.f32(&w.ln1_g, p, E);
    if ((p = L.get(q + "ln1.bias", {(uint32_t)E}))) B.f32(&w.ln1_b, p, E);
    if ((p = L.get(q + "ff.linear1.weight", {(uint32_t)c.tf_ff, (uint32_t)E}))) B.actp(&w.w1, p, (size_t)c.tf_ff * E);
    if ((p = L.get(q + "ff.linear1.bias", {(uint32_t)c.tf_ff}))) B.f32(&w.b1, p, c.tf_ff);
    if ((p = L.get(q + "ff.linear2.weight", {(uint32_t)E, (uint32_t)c.tf_ff}))) B.actp(&w.w2, p, (size_t)c.tf_ff * E);
    if ((p = L.get(q + "ff.linear2.bias", {(uint32_t)E}))) B.f32(&w.b2, p, E);
    if ((p = L.get(q + "ln2.weight", {(uint32_t)E}))) B.f32(&w.ln2_g, p, E);
    if ((p = L.get(q + "ln2.bias", {(uint32_t)E}))) B.f32(&w.ln2_b, p, E);
  }
  if ((p = L.get("head.fc1.weight", {(uint32_t)E, (uint32_t)E}))) B.actp(&W.head_w1, p, (size_t)E * E);
  if ((p = L.get("head.fc1.bias", {(uint32_t)E}))) B.f32(&W.head_b1, p, E);
  if ((p = L.get("head.fc2.weight", {(uint32_t)c.n_spk, (uint32_t)E}))) B.f32(&W.head_w2, p, (size_t)c.n_spk * E);
  if ((p = L.get("head.fc2.bias", {(uint32_t)c.n_spk}))) B.f32(&W.head_b2, p, c.n_spk);
  if (!L.err.empty()) return fail(e, SF_EFORMAT, L.err);

  cudaError_t ce = cudaMalloc(&e->d_weights, arena.host.size());
  if (ce != cudaSuccess) return cuda_fail(e, ce, "weights");
  ce = cudaMemcpy(e->d_weights, arena.host.data(), arena.host.size(), cudaMemcpyHostToDevice);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "weights upload");
  for (auto& f : arena.fix) *f.first = static_cast<uint8_t*>(e->d_weights) + f.second;

  // relative-position tables: P_l = pe . W_pos_l^T for r = -(R-1) .. R-1
  const int R = e->R, NR = 2 * R - 1;
  std::vector<float> pe((size_t)NR * D);
  for (int i = 0; i < NR; ++i) {
    const double r = (double)(i - (R - 1));
    for (int m2 = 0; m2 < D / 2; ++m2) {
      const double ang = r * pow(10000.0, -2.0 * m2 / D);
      pe[(size_t)i * D + 2 * m2] = (float)sin(ang);
      pe[(size_t)i * D + 2 * m2 + 1] = (float)cos(ang);
    }
  }
  std::vector<uint8_t> pe_act;
  to_act<T>(pe, pe_act);
  void* d_pe = nullptr;
  void* d_wpos = nullptr;
  const size_t tab_bytes = (size_t)NR * D * sizeof(T);
  ce = cudaMalloc(&e->d_ptab, tab_bytes * c.n_conformer);
  if (ce == cudaSuccess) ce = cudaMalloc(&d_pe, pe_act.size());
  if (ce == cudaSuccess) ce = cudaMalloc(&d_wpos, (size_t)D * D * sizeof(T));
  if (ce == cudaSuccess) ce = cudaMemcpy(d_pe, pe_act.data(), pe_act.size(), cudaMemcpyHostToDevice);
  for (int l = 0; l < c.n_conformer && ce == cudaSuccess; ++l) {
    const float* wp = m["enc.layers." + std::to_string(l) + ".att.linear_pos.weight"].data;
    std::vector<uint8_t> wa;
    to_act<T>(vec(wp, (size_t)D * D), wa);
    ce = cudaMemcpy(d_wpos, wa.data(), wa.size(), cudaMemcpyHostToDevice);
    T* dst = reinterpret_cast<T*>(static_cast<uint8_t*>(e->d_ptab) + tab_bytes * l);
    W.conf[l].ptab = dst;
    Epi ep{};
    ep.kind = EPI_BIAS;
    ep.out = dst;
    ep.ldo = D;
    if (ce == cudaSuccess) {
      if (sizeof(T) == 4)
        ce = gemm_f32(reinterpret_cast<const float*>(d_pe), D, reinterpret_cast<const float*>(d_wpos), NR, D, D, ep, 0);
      else
        ce = gemm_bf16_mma(reinterpret_cast<const bf16*>(d_pe), D, reinterpret_cast<const bf16*>(d_wpos), NR, D, D, ep, 0);
    }
    if (ce == cudaSuccess) ce = cudaDeviceSynchronize();
  }
  if (d_pe) cudaFree(d_pe);
  if (d_wpos) cudaFree(d_wpos);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "position tables");
  return SF_OK;
}

template <typename T> Weights<T>& weights(sf_engine* e);
template <> Weights<float>& weights<float>(sf_engine* e) { return e->wf; }
template <> Weights<bf16>& weights<bf16>(sf_engine* e) { return e->wb; }

template <typename T>
cudaError_t gemm_dispatch(sf_engine* e, const T* A, int lda, const T* W, int M, int N, int K, const Epi& ep,
                          cudaStream_t st);
template <>
cudaError_t gemm_dispatch<float>(sf_engine*, const float* A, int lda, const float* W, int M, int N, int K,
                                 const Epi& ep, cudaStream_t st) {
  return gemm_f32(A, lda, W, M, N, K, ep, st);
}
template <>
cudaError_t gemm_dispatch<bf16>(sf_engine* e, const bf16* A, int lda, const bf16* W, int M, int N, int K,
                                const Epi& ep, cudaStream_t st) {
  if (e->gemm_path >= 1 && N % 16 == 0) return gemm_bf16_tc(A, lda, W, M, N, K, ep, e->tc_scratch(), st);
  return gemm_bf16_mma(A, lda, W, M, N, K, ep, st);
}

// Transformer MHSA in the bf16 engine: the tcgen05 kernel (SF_OPT_ATTN_PATH
// 1, the default), which splits each (query tile, head) unit's keys over a
// CTA cluster when the units alone leave SMs idle (one long clip); the
// mma.sync kernel (path 0).
template <typename T>
cudaError_t mha_attention(sf_engine* e, const T* qkv, T* ctx, const SeqTable* seq, int n_tiles, int M, cudaStream_t st) {
  return launch_mha<T>(qkv, ctx, seq, n_tiles, M, e->R, st);
}
template <>
cudaError_t mha_attention<bf16>(sf_engine* e, const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles, int M,
                                cudaStream_t st) {
  if (e->attn_path == 1) return launch_mha_tc(qkv, ctx, seq, e->att_tiles2, M, e->att_max_len, e->d_err, st);
  return launch_mha<bf16>(qkv, ctx, seq, n_tiles, M, e->R, st);
}

// Relative-position attention: the bf16 engine runs it on tcgen05 unless the
// mma.sync kernel is selected (SF_OPT_ATTN_PATH = 0).
template <typename T>
cudaError_t relpos_attention(sf_engine* e, const T* qkv, const T* ptab, const float* pu, const float* pv, T* ctx,
                             const SeqTable* seq, int n_tiles, int M, cudaStream_t st) {
  return launch_relpos_attention<T>(qkv, ptab, e->R, pu, pv, ctx, seq, n_tiles, M, st);
}
template <>
cudaError_t relpos_attention<bf16>(sf_engine* e, const bf16* qkv, const bf16* ptab, const float* pu, const float* pv,
                                   bf16* ctx, const SeqTable* seq, int n_tiles, int M, cudaStream_t st) {
  if (e->attn_path == 1)
    return launch_relpos_attention_tc(qkv, ptab, e->R, pu, pv, ctx, seq, e->att_tiles2, M, e->att_max_len,
                                      e->tc_scratch(), st);
  return launch_relpos_attention<bf16>(qkv, ptab, e->R, pu, pv, ctx, seq, n_tiles, M, st);
}

template <typename T>
cudaError_t gemm_acc(sf_engine* e, const T* A, int lda, const T* W, int M, int N, int K, const Epi& ep,
                     cudaStream_t st) {
  const double a = sizeof(T);
  const double out_b = (ep.kind == EPI_RESID) ? 8.0 : (ep.kind == EPI_F32 ? 4.0 : (ep.kind == EPI_F32_AND_T ? 4.0 + a : (ep.kind == EPI_BIAS_GLU ? a / 2 : a)));
  RUN(K_GEMM, 1, 2.0 * M * N * K, ((double)M * K + (double)N * K) * a + (double)M * N * out_b,
      gemm_dispatch<T>(e, A, lda, W, M, N, K, ep, st));
  return cudaSuccess;
}

Epi epi(int kind, const float* bias, void* out, int ldo, float alpha = 1.f) {
  Epi e{};
  e.kind = kind;
  e.bias = bias;
  e.out = out;
  e.ldo = ldo;
  e.alpha = alpha;
  return e;
}

// Residual projection followed by LayerNorm over each row of the f32
// residual stream x [M x N]: x_new = x + alpha (A W^T + bias); then with
// xnorm = 0: x <- x_new, h <- act(LN(x_new)); with xnorm = 1: x <- LN(x_new)
// and h <- act(LN2(x)) when g2 is given, else act(x).  One launch (the
// LayerNorm in the GEMM's epilogue, exchanged across the row block's CTA
// cluster) in bf16 engines where the shape allows it, else the projection
// and a LayerNorm kernel.
template <typename T>
cudaError_t resid_ln(sf_engine* e, const T* A, int lda, const T* W, int M, int N, int K, const float* bias,
                     float alpha, float* x, const float* g, const float* b, bool xnorm, T* h, cudaStream_t st,
                     const float* g2 = nullptr, const float* b2 = nullptr) {
  if (sizeof(T) == 2 && e->ln_fuse && e->gemm_path >= 1 && gemm_ln_fusable(M, N, K)) {
    Epi ep = epi(EPI_RESID_LN, bias, x, N, alpha);
    ep.ln_g = g;
    ep.ln_b = b;
    ep.ln_g2 = g2;
    ep.ln_b2 = b2;
    ep.ln_h = h;
    ep.ldh = N;
    ep.ln_xnorm = xnorm ? 1 : 0;
    const double a = sizeof(T);
    RUN(K_GEMM, 1, 2.0 * M * N * K, ((double)M * K + (double)N * K) * a + (double)M * N * (8.0 + a),
        gemm_dispatch<T>(e, A, lda, W, M, N, K, ep, st));
    return cudaSuccess;
  }
  CK(gemm_acc<T>(e, A, lda, W, M, N, K, epi(EPI_RESID, bias, x, N, alpha), st));
  RUN(K_LN, 1, 0, (double)M * N * (4 + sizeof(T) + (xnorm ? 4 : 0)),
      launch_layernorm<T>(x, g, b, M, N, xnorm, h, st, g2, b2));
  return cudaSuccess;
}

// ------------------------------------------------------------ descriptors
DescBlock* desc_begin(sf_engine* e) {
  if (e->desc_pending) {
    // the previous call's copy of the block must have left the pinned buffer;
    // an error here is the stream's and resurfaces at its next launch check
    cudaEventSynchronize(e->desc_ev);
    e->desc_pending = false;
  }
  return e->h_desc;
}
cudaError_t desc_upload(sf_engine* e, cudaStream_t st) {
  CK(cudaMemcpyAsync(e->d_desc, e->h_desc, sizeof(DescBlock), cudaMemcpyHostToDevice, st));
  if (!e->capturing) {   // a graph replay records the event after its launch (run_graph)
    CK(cudaEventRecord(e->desc_ev, st));
    e->desc_pending = true;
  }
  return cudaSuccess;
}
void destroy_graphs(sf_engine* e) {
  for (auto& kv : e->graphs) {
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
    for (cudaEvent_t ev : kv.second.events) cudaEventDestroy(ev);
  }
  e->graphs.clear();
}

// Graphs whose key starts with `prefix` (e.g. every graph of one stream).
void destroy_graphs_with_prefix(sf_engine* e, const std::string& prefix) {
  for (auto it = e->graphs.begin(); it != e->graphs.end();) {
    if (it->first.compare(0, prefix.size(), prefix) == 0) {
      if (it->second.exec) cudaGraphExecDestroy(it->second.exec);
      for (cudaEvent_t ev : it->second.events) cudaEventDestroy(ev);
      it = e->graphs.erase(it);
    } else {
      ++it;
    }
  }
}

std::string stream_graph_prefix(const sf_stream* s) { return "st|" + std::to_string(s->serial) + "|"; }

// Runs `enqueue` (which must only enqueue work on `st`: no allocation, no
// synchronisation) through a CUDA graph cached under `key`: captured on
// first use (or after the workspace moved), replayed afterwards.  Launch
// counters of a replay are those recorded at capture; with profiling on,
// the graph carries its own event pairs, read back after each replay.
template <typename F>
cudaError_t run_graph(sf_engine* e, std::string key, cudaStream_t st, F&& enqueue) {
  if (!e->use_graphs) return enqueue(st);
  key += e->prof ? "|p" + std::to_string(e->prof_mask) : "|n";
  key += e->use_pdl ? "|pdl" : "";
  key += "|g" + std::to_string(e->gemm_path) + "." + std::to_string(e->pair_bn) + "|a" + std::to_string(e->attn_path) +
         "|m" + std::to_string(e->mel_path) + "|s" + std::to_string(e->sub_path) + "|n" + std::to_string(e->ln_fuse) + "|t" + std::to_string(e->tf_fuse);
  auto it = e->graphs.find(key);
  if (it != e->graphs.end() && it->second.gen != e->ws_gen) {
    cudaGraphExecDestroy(it->second.exec);
    for (cudaEvent_t ev : it->second.events) cudaEventDestroy(ev);
    e->graphs.erase(it);
    it = e->graphs.end();
  }
  if (it == e->graphs.end()) {
    if (e->graphs.size() >= 256) destroy_graphs(e);
    sf_engine::GraphEntry g;
    int64_t l0[K_COUNT];
    double f0[K_COUNT], b0[K_COUNT];
    memcpy(l0, e->launches, sizeof(l0));
    memcpy(f0, e->kflops, sizeof(f0));
    memcpy(b0, e->kbytes, sizeof(b0));
    std::vector<ProfRec> saved;
    saved.swap(e->recs);
    e->cap_events.clear();
    e->capturing = true;
    cudaError_t err = cudaStreamBeginCapture(e->cap_stream, cudaStreamCaptureModeThreadLocal);
    if (err != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
    if (err == cudaSuccess) {
      cudaError_t qe = enqueue(e->cap_stream);
      cudaGraph_t graph = nullptr;
      err = cudaStreamEndCapture(e->cap_stream, &graph);
      if (err != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
      if (qe != cudaSuccess) err = qe;
      if (err == cudaSuccess) {
        err = cudaGraphInstantiate(&g.exec, graph, 0);
        if (err != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
      }
      if (graph) cudaGraphDestroy(graph);
    }
    e->capturing = false;
    g.recs.swap(e->recs);
    e->recs.swap(saved);
    g.events.swap(e->cap_events);
    for (int k = 0; k < K_COUNT; ++k) {
      g.launches[k] = e->launches[k] - l0[k];
      g.flops[k] = e->kflops[k] - f0[k];
      g.bytes[k] = e->kbytes[k] - b0[k];
    }
    memcpy(e->launches, l0, sizeof(l0));
    memcpy(e->kflops, f0, sizeof(f0));
    memcpy(e->kbytes, b0, sizeof(b0));
    if (err != cudaSuccess) {
      for (cudaEvent_t ev : g.events) cudaEventDestroy(ev);
      cudaGetLastError();
      return err;
    }
    g.gen = e->ws_gen;
    it = e->graphs.emplace(key, std::move(g)).first;
  }
  sf_engine::GraphEntry& g = it->second;
  CK(cudaGraphLaunch(g.exec, st));
  CK(cudaEventRecord(e->desc_ev, st));
  e->desc_pending = true;
  for (int k = 0; k < K_COUNT; ++k) {
    e->launches[k] += g.launches[k];
    e->kflops[k] += g.flops[k];
    e->kbytes[k] += g.bytes[k];
  }
  if (e->prof && !g.recs.empty()) {
    CK(cudaStreamSynchronize(st));
    for (const ProfRec& r : g.recs) {
      float t = 0.f;
      CK(cudaEventElapsedTime(&t, r.a, r.b));
      e->ms_acc[r.cls] += t;
    }
  }
  return cudaSuccess;
}

// Fill the sequence table from lengths; returns total rows and tile count.
double sum_sq(const std::vector<int>& lens) {
  double s2 = 0;
  for (int v : lens) s2 += (double)v * v;
  return s2;
}
void fill_seq(DescBlock* d, const std::vector<int>& lens, int& M, int& tiles) {
  d->seq.n_seq = (int)lens.size();
  M = 0;
  tiles = 0;
  int tiles2 = 0;
  for (size_t i = 0; i < lens.size(); ++i) {
    d->seq.off[i] = M;
    d->seq.tile_off[i] = tiles;
    d->seq.tile2_off[i] = tiles2;
    M += lens[i];
    tiles += (lens[i] + ATT_TILE - 1) / ATT_TILE;
    tiles2 += (lens[i] + 2 * ATT_TILE - 1) / (2 * ATT_TILE);
  }
  d->seq.off[lens.size()] = M;
  d->seq.tile_off[lens.size()] = tiles;
  d->seq.tile2_off[lens.size()] = tiles2;
  d->seq.total = M;
}

// -------------------------------------------------------------- pipeline
// ConvSubsampling of n_win windows (PreArgs in the descriptor) -> act
// embeddings; output row (i, t) goes to out + (i * out_stride + t) * D.
// Workspace of run_pre_encode (call before any capture).
cudaError_t prep_pre_encode(sf_engine* e, int n_win, int64_t W_max, size_t a) {
  const int T1 = (int)half_len(W_max), T2 = (int)half_len(T1), T3 = (int)half_len(T2);
  if (e->sub_path == 0) CK(ensure(e->sub1, (size_t)n_win * T1 * 64 * 256 * a));   // path 1 keeps stage 1 on chip
  CK(ensure(e->sub2a, (size_t)n_win * T2 * 32 * 256 * a));
  CK(ensure(e->sub2b, (size_t)n_win * T2 * 32 * 256 * a));
  CK(ensure(e->sub3a, (size_t)n_win * T3 * 16 * 256 * a));
  CK(ensure(e->sub3b, (size_t)n_win * T3 * 16 * 256 * a));
  return cudaSuccess;
}

template <typename T>
cudaError_t run_pre_encode(sf_engine* e, const float* feats, int64_t t_buf, int n_win, int64_t W_max, T* out,
                           int64_t out_stride, cudaStream_t st) {
  Weights<T>& W = weights<T>(e);
  const int D = e->cfg.d_model;
  const int T1 = (int)half_len(W_max), T2 = (int)half_len(T1), T3 = (int)half_len(T2);
  PreArgs pa{e->d_desc->buf, e->d_desc->start, e->d_desc->frames};
  T* s1 = static_cast<T*>(e->sub1.p);
  T* s2a = static_cast<T*>(e->sub2a.p);
  T* s2b = static_cast<T*>(e->sub2b.p);
  T* s3a = static_cast<T*>(e->sub3a.p);
  T* s3b = static_cast<T*>(e->sub3b.p);
  if (e->sub_path == 1) {
    RUN(K_CONV1, 1, 18.0 * 256 * (64 * T1 + 32 * T2) * n_win,
        (double)n_win * W_max * 128 * 4 + (double)n_win * T2 * 32 * 256 * sizeof(T),
        launch_conv1_dw<T>(feats, t_buf, pa, n_win, W.c1_w, W.c1_b, W.dw_w[0], W.dw_b[0], s2a, T2, st));
  } else {
    RUN(K_CONV1, 1, 18.0 * 256 * 64 * T1 * n_win,
        (double)n_win * W_max * 128 * 4 + (double)n_win * T1 * 64 * 256 * sizeof(T),
        launch_conv1<T>(feats, t_buf, pa, n_win, W.c1_w, W.c1_b, s1, T1, st));
    RUN(K_DW2D, 1, 18.0 * 256 * 32 * T2 * n_win, (double)n_win * (T1 * 64 + T2 * 32) * 256 * sizeof(T),
        launch_dwconv3x3s2<T>(s1, T1, 64, s2a, T2, 32, pa, n_win, 1, W.dw_w[0], W.dw_b[0], st));
  }
  CK(gemm_acc<T>(e, s2a, 256, W.pw_w[0], n_win * T2 * 32, 256, 256, epi(EPI_BIAS_RELU, W.pw_b[0], s2b, 256), st));
  RUN(K_DW2D, 1, 18.0 * 256 * 16 * T3 * n_win, (double)n_win * (T2 * 32 + T3 * 16) * 256 * sizeof(T),
      launch_dwconv3x3s2<T>(s2b, T2, 32, s3a, T3, 16, pa, n_win, 2, W.dw_w[1], W.dw_b[1], st));
  CK(gemm_acc<T>(e, s3a, 256, W.pw_w[1], n_win * T3 * 16, 256, 256, epi(EPI_BIAS_RELU, W.pw_b[1], s3b, 256), st));
  Epi eo = epi(EPI_BIAS, W.out_b, out, D);
  eo.rpg = T3;
  eo.gstride = out_stride;
  CK(gemm_acc<T>(e, s3b, 16 * 256, W.out_w, n_win * T3, D, 16 * 256, eo, st));
  return cudaSuccess;
}

// Encoder on the packed f32 stream in e->x (M rows): conformer layers,
// encoder_proj, transformer layers, head -> probs (M x 4 f32).
template <typename T>
cudaError_t run_encode(sf_engine* e, int M, int n_tiles, float* probs, cudaStream_t st) {
  Weights<T>& W = weights<T>(e);
  const sf_config& c = e->cfg;
  const int D = c.d_model, E = c.tf_d_model, DFF = D * c.ff_mult;
  const SeqTable* seq = &e->d_desc->seq;
  float* x = static_cast<float*>(e->x.p);
  T* h = static_cast<T*>(e->h.p);
  T* big = static_cast<T*>(e->big.p);
  T* ctx = static_cast<T*>(e->ctx.p);
  for (int l = 0; l < c.n_conformer; ++l) {
    const ConfW<T>& w = W.conf[l];
    if (l == 0)   // later layers get this LN fused into the previous layer's final LN
      RUN(K_LN, 1, 0, (double)M * D * (4 + sizeof(T)), launch_layernorm<T>(x, w.ff1_g, w.ff1_b, M, D, false, h, st));
    CK(gemm_acc<T>(e, h, D, w.ff1_w1, M, DFF, D, epi(EPI_BIAS_SWISH, w.ff1_b1, big, DFF), st));
    CK(resid_ln<T>(e, big, DFF, w.ff1_w2, M, D, DFF, w.ff1_b2, 0.5f, x, w.att_g, w.att_b, false, h, st));
    CK(gemm_acc<T>(e, h, D, w.wqkv, M, 3 * D, D, epi(EPI_BIAS, w.bqkv, big, 3 * D), st));
    RUN(K_ATT_REL, 1, 6.0 * e->att_s2 * D, (double)M * 4 * D * sizeof(T),
        relpos_attention<T>(e, big, w.ptab, w.pu, w.pv, ctx, seq, n_tiles, M, st));
    CK(resid_ln<T>(e, ctx, D, w.wo, M, D, D, w.bo, 1.f, x, w.conv_g, w.conv_b, false, h, st));
    CK(gemm_acc<T>(e, h, D, w.pw1, M, 2 * D, D, epi(EPI_BIAS_GLU, w.pw1_b, ctx, D), st));
    RUN(K_DW1D, 1, 2.0 * M * D * c.conv_kernel, (double)M * D * 2 * sizeof(T),
        launch_dwconv1d<T>(ctx, h, w.dw_w, w.dw_b, M, D, c.conv_kernel, seq, st));
    CK(resid_ln<T>(e, h, D, w.pw2, M, D, D, w.pw2_b, 1.f, x, w.ff2_g, w.ff2_b, false, h, st));
    CK(gemm_acc<T>(e, h, D, w.ff2_w1, M, DFF, D, epi(EPI_BIAS_SWISH, w.ff2_b1, big, DFF), st));
    // layer-final LN (x <- LN(x)), then the next layer's FFN1 LN into h
    const bool next = l + 1 < c.n_conformer;
    CK(resid_ln<T>(e, big, DFF, w.ff2_w2, M, D, DFF, w.ff2_b2, 0.5f, x, w.out_g, w.out_b, true, h, st,
                   next ? W.conf[l + 1].ff1_g : nullptr, next ? W.conf[l + 1].ff1_b : nullptr));
  }
  float* x2 = static_cast<float*>(e->x2.p);
  T* h2 = static_cast<T*>(e->h2.p);
  {
    Epi ep = epi(EPI_F32_AND_T, W.proj_b, x2, E);
    ep.out2 = h2;
    ep.ldo2 = E;
    CK(gemm_acc<T>(e, h, D, W.proj_w, M, E, D, ep, st));
  }
  if (sizeof(T) == 2 && e->gemm_path >= 1 && c.n_transformer > 0 && E == 192 && c.tf_ff == 768 &&
      (e->tf_fuse == 2 || (e->tf_fuse == 1 && M <= tf_layer_max_rows()))) {
    // fused layers: layer 0's Q|K|V projection, then per layer the attention
    // and one kernel for the rest of the layer and the next layer's Q|K|V
    auto tfw = [&](int l) {
      const TfW<T>& w = W.tf[l];
      return TfLayerW{reinterpret_cast<const bf16*>(w.wqkv), reinterpret_cast<const bf16*>(w.wo),
                      reinterpret_cast<const bf16*>(w.w1), reinterpret_cast<const bf16*>(w.w2), w.bqkv, w.bo,
                      w.ln1_g, w.ln1_b, w.b1, w.b2, w.ln2_g, w.ln2_b};
    };
    CK(gemm_acc<T>(e, h2, E, W.tf[0].wqkv, M, 3 * E, E, epi(EPI_BIAS, W.tf[0].bqkv, big, 3 * E), st));
    for (int l = 0; l < c.n_transformer; ++l) {
      const bool next = l + 1 < c.n_transformer;
      RUN(K_ATT_MHA, 1, 4.0 * e->att_s2 * E, (double)M * 4 * E * sizeof(T),
          mha_attention<T>(e, big, ctx, seq, n_tiles, M, st));
      const TfLayerW cur = tfw(l), nxt = next ? tfw(l + 1) : TfLayerW{};
      RUN(K_TFL, 1, 2.0 * M * E * (E + 2.0 * c.tf_ff + (next ? 3.0 * E : 0.0)),
          (double)M * (E * sizeof(T) + 8.0 * E + (next ? 3.0 * E : E) * sizeof(T)),
          launch_tf_layer(reinterpret_cast<const bf16*>(ctx), cur, next ? &nxt : nullptr, x2,
                          reinterpret_cast<bf16*>(big), reinterpret_cast<bf16*>(h2), M, e->d_err, st));
    }
  } else {
  for (int l = 0; l < c.n_transformer; ++l) {
    const TfW<T>& w = W.tf[l];
    CK(gemm_acc<T>(e, h2, E, w.wqkv, M, 3 * E, E, epi(EPI_BIAS, w.bqkv, big, 3 * E), st));
    RUN(K_ATT_MHA, 1, 4.0 * e->att_s2 * E, (double)M * 4 * E * sizeof(T), mha_attention<T>(e, big, ctx, seq, n_tiles, M, st));
    CK(resid_ln<T>(e, ctx, E, w.wo, M, E, E, w.bo, 1.f, x2, w.ln1_g, w.ln1_b, true, h2, st));
    CK(gemm_acc<T>(e, h2, E, w.w1, M, c.tf_ff, E, epi(EPI_BIAS_RELU, w.b1, big, c.tf_ff), st));
    CK(resid_ln<T>(e, big, c.tf_ff, w.w2, M, E, c.tf_ff, w.b2, 1.f, x2, w.ln2_g, w.ln2_b, true, h2, st));
  }
  }
  CK(gemm_acc<T>(e, h2, E, W.head_w1, M, E, E, epi(EPI_BIAS_RELU, W.head_b1, ctx, E), st));
  RUN(K_HEAD, 1, 2.0 * M * E * 4, (double)M * (E * sizeof(T) + 16), launch_head_out<T>(ctx, W.head_w2, W.head_b2, probs, M, E, st));
  return cudaSuccess;
}

cudaError_t ensure_encode_ws(sf_engine* e, int M) {
  const size_t a = act_size(e);
  const int D = e->cfg.d_model, E = e->cfg.tf_d_model;
  const size_t big_cols = std::max<size_t>({(size_t)D * e->cfg.ff_mult, (size_t)3 * D, (size_t)e->cfg.tf_ff});
  CK(ensure(e->x, (size_t)M * D * 4));
  CK(ensure(e->h, (size_t)M * D * a));
  CK(ensure(e->big, (size_t)M * big_cols * a));
  CK(ensure(e->ctx, (size_t)M * D * a));
  CK(ensure(e->x2, (size_t)M * E * 4));
  CK(ensure(e->h2, (size_t)M * E * a));
  CK(ensure(e->probs, (size_t)M * 4 * 4));
  return cudaSuccess;
}

template <typename T>
cudaError_t offline_impl(sf_engine* e, const float* d_audio, const std::vector<int64_t>& len, int B, int64_t n_max,
                         float* d_probs, cudaStream_t st) {
  DescBlock* d = desc_begin(e);
  const int64_t T_cols = 1 + n_max / 160;
  std::vector<int> tp(B);
  int64_t L_max = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t L = len[b] / 160;
    d->len[b] = len[b];
    d->buf[b] = b;
    d->start[b] = 0;
    d->frames[b] = L;
    tp[b] = (int)enc_frames(L);
    L_max = std::max(L_max, L);
    d->step.stream[b] = b;
    d->step.n_c[b] = d->step.n_f[b] = d->step.lc[b] = 0;
    d->step.cur_c[b] = d->step.cur_f[b] = 0;
  }
  int M, tiles;
  fill_seq(d, tp, M, tiles);
  e->att_s2 = sum_sq(tp);
  e->att_tiles2 = d->seq.tile2_off[d->seq.n_seq];
  e->att_max_len = 0;
  for (int q_ = 0; q_ < d->seq.n_seq; ++q_)
    e->att_max_len = std::max(e->att_max_len, d->seq.off[q_ + 1] - d->seq.off[q_]);
  const int T3 = (int)enc_frames(L_max);
  const int Tp_max = (int)enc_frames(n_max / 160);
  CK(ensure(e->mel, (size_t)B * 128 * T_cols * 4));
  CK(ensure(e->part, mel_part_floats(B, n_max) * 4));
  CK(ensure(e->emb, (size_t)B * T3 * e->cfg.d_model * sizeof(T)));
  CK(ensure_encode_ws(e, M));
  CK(prep_pre_encode(e, B, L_max, sizeof(T)));
  std::string key = "off|" + std::to_string(B) + "|" + std::to_string(n_max) + "|" +
                    std::to_string(reinterpret_cast<uintptr_t>(d_audio)) + "|" +
                    std::to_string(reinterpret_cast<uintptr_t>(d_probs));
  for (int b = 0; b < B; ++b) key += "|" + std::to_string(len[b]);
  return run_graph(e, key, st, [&](cudaStream_t st) -> cudaError_t {
    CK(desc_upload(e, st));
    MelArgs ma{e->d_desc->len};
    RUN(K_MEL, e->mel_path ? 3 : 2, 0, (double)B * n_max * 4 + (double)B * 128 * T_cols * 4,
        launch_mel(d_audio, B, n_max, ma, e->d_mel_tab, static_cast<float*>(e->mel.p), static_cast<float*>(e->part.p), st,
                   e->mel_path));
    CK(run_pre_encode<T>(e, static_cast<float*>(e->mel.p), T_cols, B, L_max, static_cast<T*>(e->emb.p), T3, st));
    StateBufs none{};
    none.D = e->cfg.d_model;
    RUN(K_ASSEMBLE, 1, 0, (double)M * e->cfg.d_model * (4 + sizeof(T)),
        launch_assemble<T>(static_cast<float*>(e->x.p), &e->d_desc->seq, &e->d_desc->step, none,
                           static_cast<T*>(e->emb.p), T3, M, st));
    CK(run_encode<T>(e, M, tiles, static_cast<float*>(e->probs.p), st));
    RUN(K_EXTRACT, 1, 0, (double)M * 16 + (double)B * Tp_max * 16,
        launch_extract_rows(static_cast<float*>(e->probs.p), &e->d_desc->seq, nullptr, nullptr, nullptr, B, d_probs,
                            Tp_max, st));
    return cudaSuccess;
  });
}

sf_status check_engine(sf_engine* e) {
  if (!e) return SF_EINVAL;
  g_ws_gen = &e->ws_gen;
  g_fail_line = 0;
  sf::g_launch_pdl = e->use_pdl;
  sf::g_gemm_pairs = e->gemm_path == 2 ? 2 : e->gemm_path == 3 ? 0 : 1;
  sf::g_gemm_pair_bn = e->pair_bn;
  cudaGetLastError();   // start each call without a stale, non-sticky error
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != e->device) cudaSetDevice(e->device);
  return SF_OK;
}

sf_status check_offline_args(sf_engine* e, const void* audio, const int64_t* h_len, int B, int64_t n_max,
                             const void* out, std::vector<int64_t>& len) {
  if (!audio || !h_len || !out) return fail(e, SF_EINVAL, "null pointer argument");
  if (B < 1 || B > e->cfg.max_batch) return fail(e, SF_ESHAPE, "batch size out of range [1, max_batch]");
  if (n_max < 1600 || n_max > e->cfg.max_samples) return fail(e, SF_ESHAPE, "n_max out of range [1600, max_samples]");
  len.assign(h_len, h_len + B);
  for (int b = 0; b < B; ++b)
    if (len[b] < 1600 || len[b] > n_max)
      return fail(e, SF_EINVAL, "clip length must be in [1600, n_max] samples (clip " + std::to_string(b) + ")");
  return SF_OK;
}

}  // namespace

// ======================================================================= API
extern "C" {

const char* sf_status_str(sf_status s) {
  switch (s) {
    case SF_OK: return "ok";
    case SF_EINVAL: return "invalid argument";
    case SF_ESHAPE: return "size out of range";
    case SF_ENOMEM: return "out of memory";
    case SF_ECUDA: return "CUDA error";
    case SF_ESTATE: return "invalid state";
    case SF_ETIMEOUT: return "device wait timed out";
    case SF_EDEVICE: return "no usable device";
    case SF_EFORMAT: return "bad weight blob";
  }
  return "unknown status";
}

sf_status sf_default_config(sf_config* c) {
  if (!c) return SF_EINVAL;
  memset(c, 0, sizeof(*c));
  c->sample_rate = 16000;
  c->n_mels = 128;
  c->n_fft = 512;
  c->win_length = 400;
  c->hop_length = 160;
  c->subsampling = 8;
  c->d_model = 512;
  c->tf_d_model = 192;
  c->n_conformer = 17;
  c->n_transformer = 18;
  c->n_heads = 8;
  c->ff_mult = 4;
  c->tf_ff = 768;
  c->conv_kernel = 9;
  c->n_spk = 4;
  c->spkcache_len = 188;
  c->precision = SF_BF16;
  c->max_batch = 64;
  c->max_samples = 1920000;
  return SF_OK;
}

sf_status sf_create(const void* blob, uint64_t nbytes, const sf_config* cfg, sf_engine** out) {
  if (!blob || !cfg || !out) return SF_EINVAL;
  *out = nullptr;
  sf_config ref;
  sf_default_config(&ref);
  if (cfg->sample_rate != ref.sample_rate || cfg->n_mels != ref.n_mels || cfg->n_fft != ref.n_fft ||
      cfg->win_length != ref.win_length || cfg->hop_length != ref.hop_length || cfg->subsampling != ref.subsampling ||
      cfg->d_model != ref.d_model || cfg->tf_d_model != ref.tf_d_model || cfg->n_heads != ref.n_heads ||
      cfg->ff_mult != ref.ff_mult || cfg->tf_ff != ref.tf_ff || cfg->conv_kernel != ref.conv_kernel ||
      cfg->n_spk != ref.n_spk || cfg->spkcache_len != ref.spkcache_len)
    return SF_EINVAL;
  if (cfg->n_conformer < 1 || cfg->n_conformer > 64 || cfg->n_transformer < 0 || cfg->n_transformer > 64 ||
      (cfg->precision != SF_FP32 && cfg->precision != SF_BF16) || cfg->max_batch < 1 || cfg->max_batch > MAX_SEQ ||
      cfg->max_samples < 1600 || cfg->max_samples > 16000LL * 3600 * 4)
    return SF_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SF_EDEVICE;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10) return SF_EDEVICE;
  std::unique_ptr<sf_engine> e(new sf_engine());
  e->cfg = *cfg;
  e->device = dev;
  {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) e->n_sms = n;
  }
  e->R = (int)std::max<int64_t>(enc_frames(cfg->max_samples / 160), 188 + 188 + 340 + 40);
  e->max_seq_len = e->R;
  if (cfg->precision == SF_FP32 && e->R > attention_f32_max_seq()) return SF_ESHAPE;
  cudaError_t ce;
  if ((ce = gemm_init_attributes()) != cudaSuccess) return cuda_fail(e.get(), ce, "init"), SF_ECUDA;
  if ((ce = attention_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if ((ce = attention_tc_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if ((ce = attention_mha_tc_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if ((ce = gemm_tc_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if ((ce = frontend_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if ((ce = tf_layer_init_attributes()) != cudaSuccess) return SF_ECUDA;
  if (cfg->precision == SF_FP32 && (ce = attention_reserve_f32(e->R)) != cudaSuccess) return SF_ECUDA;
  g_ws_gen = &e->ws_gen;
  std::unordered_map<std::string, TensorRef> m;
  std::string err;
  if (!parse_blob(blob, nbytes, m, err)) return SF_EFORMAT;
  sf_status s = cfg->precision == SF_BF16 ? load_weights<bf16>(e.get(), m, e->wb) : load_weights<float>(e.get(), m, e->wf);
  if (s != SF_OK) {
    fprintf(stderr, "sf_create: %s\n", e->err.c_str());
    sf_destroy(e.release());
    return s;
  }
  MelTables tab;
  build_mel_tables(&tab);
  if (cudaMalloc(&e->d_mel_tab, sizeof(MelTables)) != cudaSuccess ||
      cudaMemcpy(e->d_mel_tab, &tab, sizeof(MelTables), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMallocHost(&e->h_desc, sizeof(DescBlock)) != cudaSuccess ||
      cudaMalloc(&e->d_desc, sizeof(DescBlock)) != cudaSuccess ||
      cudaEventCreateWithFlags(&e->desc_ev, cudaEventDisableTiming) != cudaSuccess ||
      cudaMalloc(&e->d_err, sizeof(int)) != cudaSuccess || cudaMemset(e->d_err, 0, sizeof(int)) != cudaSuccess ||
      cudaMalloc(&e->d_split_ws, SPLIT_WS_BYTES) != cudaSuccess ||
      cudaMalloc(&e->d_split_cnt, SPLIT_CNT * sizeof(int)) != cudaSuccess ||
      cudaMemset(e->d_split_cnt, 0, SPLIT_CNT * sizeof(int)) != cudaSuccess) {
    sf_destroy(e.release());
    return SF_ENOMEM;
  }
  memset(e->h_desc, 0, sizeof(DescBlock));
  if (cudaStreamCreateWithFlags(&e->cap_stream, cudaStreamNonBlocking) != cudaSuccess) {
    sf_destroy(e.release());
    return SF_ECUDA;
  }
  *out = e.release();
  return SF_OK;
}

sf_status sf_create_from_file(const char* path, const sf_config* cfg, sf_engine** out) {
  if (!path) return SF_EINVAL;
  FILE* f = fopen(path, "rb");
  if (!f) return SF_EINVAL;
  fseek(f, 0, SEEK_END);
  long n = ftell(f);
  fseek(f, 0, SEEK_SET);
  std::vector<uint8_t> buf(n > 0 ? n : 0);
  size_t got = n > 0 ? fread(buf.data(), 1, n, f) : 0;
  fclose(f);
  if ((long)got != n) return SF_EFORMAT;
  return sf_create(buf.data(), buf.size(), cfg, out);
}

sf_status sf_destroy(sf_engine* e) {
  if (!e) return SF_EINVAL;
  cudaDeviceSynchronize();
  for (sf_stream* s : e->streams) s->e = nullptr;   // they can still be destroyed, not stepped
  destroy_graphs(e);
  for (Buf* b : {&e->mel, &e->part, &e->audio, &e->sub1, &e->sub2a, &e->sub2b, &e->sub3a, &e->sub3b, &e->emb, &e->x,
                 &e->h, &e->big, &e->ctx, &e->x2, &e->h2, &e->probs, &e->out})
    if (b->p) cudaFree(b->p);
  if (e->d_weights) cudaFree(e->d_weights);
  if (e->d_ptab) cudaFree(e->d_ptab);
  if (e->d_mel_tab) cudaFree(e->d_mel_tab);
  if (e->d_desc) cudaFree(e->d_desc);
  if (e->h_desc) cudaFreeHost(e->h_desc);
  if (e->desc_ev) cudaEventDestroy(e->desc_ev);
  for (cudaEvent_t ev : e->pool) cudaEventDestroy(ev);
  if (e->cap_stream) cudaStreamDestroy(e->cap_stream);
  if (e->d_err) cudaFree(e->d_err);
  if (e->d_split_ws) cudaFree(e->d_split_ws);
  if (e->d_split_cnt) cudaFree(e->d_split_cnt);
  delete e;
  return SF_OK;
}

sf_status sf_get_metadata(const sf_engine* e, sf_config* out) {
  if (!e || !out) return SF_EINVAL;
  *out = e->cfg;
  return SF_OK;
}

const char* sf_last_error(const sf_engine* e) { return e ? e->err.c_str() : "null engine"; }

sf_status sf_mel(sf_engine* e, const float* d_audio, const int64_t* h_len, int B, int64_t n_max, float* d_mel,
                 int64_t* h_mel_len, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  std::vector<int64_t> len;
  sf_status s = check_offline_args(e, d_audio, h_len, B, n_max, d_mel, len);
  if (s != SF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  DescBlock* d = desc_begin(e);
  for (int b = 0; b < B; ++b) d->len[b] = len[b];
  cudaError_t ce = ensure(e->part, mel_part_floats(B, n_max) * 4);
  if (ce == cudaSuccess) ce = desc_upload(e, st);
  MelArgs ma{e->d_desc->len};
  if (ce == cudaSuccess) {
    Scope sc(e, K_MEL, e->mel_path ? 3 : 2, 0, (double)B * n_max * 4 + (double)B * 128 * (1 + n_max / 160) * 4, st);
    ce = launch_mel(d_audio, B, n_max, ma, e->d_mel_tab, d_mel, static_cast<float*>(e->part.p), st, e->mel_path);
  }
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_mel");
  if (h_mel_len)
    for (int b = 0; b < B; ++b) h_mel_len[b] = len[b] / 160;
  return SF_OK;
}

sf_status sf_forward_offline(sf_engine* e, const float* d_audio, const int64_t* h_len, int B, int64_t n_max,
                             float* d_probs, int64_t* h_out_len, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  std::vector<int64_t> len;
  sf_status s = check_offline_args(e, d_audio, h_len, B, n_max, d_probs, len);
  if (s != SF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = e->cfg.precision == SF_BF16 ? offline_impl<bf16>(e, d_audio, len, B, n_max, d_probs, st)
                                               : offline_impl<float>(e, d_audio, len, B, n_max, d_probs, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_forward_offline");
  if (h_out_len)
    for (int b = 0; b < B; ++b) h_out_len[b] = enc_frames(len[b] / 160);
  return SF_OK;
}

sf_status sf_forward_offline_host(sf_engine* e, const float* h_audio, const int64_t* h_len, int B, int64_t n_max,
                                  float* h_probs, int64_t* h_out_len, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  std::vector<int64_t> len;
  sf_status s = check_offline_args(e, h_audio, h_len, B, n_max, h_probs, len);
  if (s != SF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const int64_t Tp = enc_frames(n_max / 160);
  const size_t out_bytes = (size_t)B * Tp * 4 * 4;
  cudaError_t ce = ensure(e->audio, (size_t)B * n_max * 4);
  if (ce == cudaSuccess) ce = ensure(e->out, out_bytes);
  if (ce != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
  if (ce == cudaSuccess) ce = cudaMemcpyAsync(e->audio.p, h_audio, (size_t)B * n_max * 4, cudaMemcpyHostToDevice, st);
  if (ce != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
  if (ce == cudaSuccess)
    ce = e->cfg.precision == SF_BF16
             ? offline_impl<bf16>(e, static_cast<float*>(e->audio.p), len, B, n_max, static_cast<float*>(e->out.p), st)
             : offline_impl<float>(e, static_cast<float*>(e->audio.p), len, B, n_max, static_cast<float*>(e->out.p), st);
  if (ce == cudaSuccess) {
    ce = cudaMemcpyAsync(h_probs, e->out.p, out_bytes, cudaMemcpyDeviceToHost, st);
    if (ce != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
  }
  if (ce == cudaSuccess) {
    ce = cudaStreamSynchronize(st);
    if (ce != cudaSuccess && !g_fail_line) g_fail_line = __LINE__;
  }
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_forward_offline_host");
  if (h_out_len)
    for (int b = 0; b < B; ++b) h_out_len[b] = enc_frames(len[b] / 160);
  return SF_OK;
}

sf_status sf_pre_encode(sf_engine* e, const float* d_feats, int n_buf, int64_t t_buf, const int* h_buf,
                        const int64_t* h_start, const int64_t* h_frames, int n, void* d_embs, int64_t emb_stride,
                        void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_feats || !h_buf || !h_start || !h_frames || !d_embs) return fail(e, SF_EINVAL, "null pointer argument");
  if (n < 1 || n > MAX_SEQ || n_buf < 1 || t_buf < 1) return fail(e, SF_ESHAPE, "window count or buffer size out of range");
  DescBlock* d = desc_begin(e);
  int64_t W_max = 0;
  for (int i = 0; i < n; ++i) {
    if (h_buf[i] < 0 || h_buf[i] >= n_buf || h_start[i] < 0 || h_frames[i] < 1 || h_start[i] + h_frames[i] > t_buf)
      return fail(e, SF_ESHAPE, "window " + std::to_string(i) + " outside the feature buffer");
    if (enc_frames(h_frames[i]) > emb_stride) return fail(e, SF_ESHAPE, "emb_stride smaller than a window's output");
    d->buf[i] = h_buf[i];
    d->start[i] = h_start[i];
    d->frames[i] = h_frames[i];
    W_max = std::max(W_max, h_frames[i]);
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = prep_pre_encode(e, n, W_max, act_size(e));
  if (ce == cudaSuccess) ce = desc_upload(e, st);
  if (ce == cudaSuccess)
    ce = e->cfg.precision == SF_BF16
             ? run_pre_encode<bf16>(e, d_feats, t_buf, n, W_max, static_cast<bf16*>(d_embs), emb_stride, st)
             : run_pre_encode<float>(e, d_feats, t_buf, n, W_max, static_cast<float*>(d_embs), emb_stride, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_pre_encode");
  return SF_OK;
}

sf_status sf_encode(sf_engine* e, const void* d_embs, const int* h_seq_len, int n, float* d_preds, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_embs || !h_seq_len || !d_preds) return fail(e, SF_EINVAL, "null pointer argument");
  if (n < 1 || n > MAX_SEQ) return fail(e, SF_ESHAPE, "sequence count out of range");
  std::vector<int> lens(h_seq_len, h_seq_len + n);
  for (int v : lens)
    if (v < 1 || v > e->max_seq_len) return fail(e, SF_ESHAPE, "sequence length out of range");
  DescBlock* d = desc_begin(e);
  int M, tiles;
  fill_seq(d, lens, M, tiles);
  e->att_s2 = sum_sq(lens);
  e->att_tiles2 = d->seq.tile2_off[d->seq.n_seq];
  e->att_max_len = 0;
  for (int q_ = 0; q_ < d->seq.n_seq; ++q_)
    e->att_max_len = std::max(e->att_max_len, d->seq.off[q_ + 1] - d->seq.off[q_]);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = ensure_encode_ws(e, M);
  if (ce == cudaSuccess) ce = desc_upload(e, st);
  const int64_t nel = (int64_t)M * e->cfg.d_model;
  if (ce == cudaSuccess) {
    Scope sc(e, K_TOF32, 1, 0, (double)nel * (4 + act_size(e)), st);
    ce = e->cfg.precision == SF_BF16 ? launch_to_f32<bf16>(static_cast<const bf16*>(d_embs), static_cast<float*>(e->x.p), nel, st)
                                     : launch_to_f32<float>(static_cast<const float*>(d_embs), static_cast<float*>(e->x.p), nel, st);
  }
  if (ce == cudaSuccess)
    ce = e->cfg.precision == SF_BF16 ? run_encode<bf16>(e, M, tiles, d_preds, st) : run_encode<float>(e, M, tiles, d_preds, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_encode");
  return SF_OK;
}

sf_status sf_check(sf_engine* e, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  cudaError_t ce = cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream));
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_check");
  int w = 0;
  ce = cudaMemcpy(&w, e->d_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (ce == cudaSuccess && w) ce = cudaMemset(e->d_err, 0, sizeof(int));
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_check");
  if (w & ERR_TIMEOUT) return fail(e, SF_ETIMEOUT, "a bounded device wait gave up");
  if (w) return fail(e, SF_EDEVICE, "a device-side check failed (error word " + std::to_string(w) + ")");
  return SF_OK;
}

sf_status sf_selftest_wait(sf_engine* e, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  cudaError_t ce = launch_selftest_wait(e->d_err, static_cast<cudaStream_t>(cuda_stream));
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_selftest_wait");
  return SF_OK;
}

sf_status sf_gemm_bf16(sf_engine* e, const void* d_A, int lda, const void* d_W, int M, int N, int K,
                       const float* d_bias, void* d_C, int path, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_A || !d_W || !d_C) return fail(e, SF_EINVAL, "null pointer argument");
  if (M < 1 || N < 16 || K < 64 || N % 16 || K % 64 || lda < K || lda % 8 || path < 0 || path > 5)
    return fail(e, SF_ESHAPE, "sf_gemm_bf16: M >= 1, N % 16 == 0, K % 64 == 0, lda >= K, lda % 8 == 0, path 0..5");
  static const int kinds[6] = {EPI_F32, EPI_F32, EPI_BIAS, EPI_RESID, EPI_BIAS_SWISH, EPI_BIAS_GLU};
  Epi ep = epi(kinds[path], d_bias, d_C, path == 5 ? N / 2 : N);
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const bf16* A = static_cast<const bf16*>(d_A);
  const bf16* W = static_cast<const bf16*>(d_W);
  cudaError_t ce = path >= 1 ? gemm_bf16_tc(A, lda, W, M, N, K, ep, e->tc_scratch(), st)
                             : gemm_bf16_mma(A, lda, W, M, N, K, ep, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_gemm_bf16");
  return SF_OK;
}

sf_status sf_gemm_bf16_ln(sf_engine* e, const void* d_A, int lda, const void* d_W, int M, int N, int K,
                          const float* d_bias, float alpha, float* d_x, const float* d_g, const float* d_b,
                          const float* d_g2, const float* d_b2, int xnorm, void* d_h, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_A || !d_W || !d_x || !d_g || !d_b || !d_h || (d_g2 && !d_b2)) return fail(e, SF_EINVAL, "null pointer argument");
  if (d_g2 && !xnorm) return fail(e, SF_EINVAL, "a second LayerNorm needs xnorm = 1");
  if (e->cfg.precision != SF_BF16) return fail(e, SF_ESTATE, "sf_gemm_bf16_ln needs a bf16 engine");
  if (M < 1 || K < 64 || K % 64 || lda < K || lda % 8 || !gemm_ln_fusable(M, N, K))
    return fail(e, SF_ESHAPE, "sf_gemm_bf16_ln: N a multiple of 64 up to 512, one wave of row blocks, K % 64 == 0");
  if ((reinterpret_cast<uintptr_t>(d_x) & 15) || (reinterpret_cast<uintptr_t>(d_h) & 7))
    return fail(e, SF_EINVAL, "x must be 16-byte and h 8-byte aligned");
  Epi ep = epi(EPI_RESID_LN, d_bias, d_x, N, alpha);
  ep.ln_g = d_g;
  ep.ln_b = d_b;
  ep.ln_g2 = d_g2;
  ep.ln_b2 = d_b2;
  ep.ln_h = d_h;
  ep.ldh = N;
  ep.ln_xnorm = xnorm ? 1 : 0;
  cudaError_t ce = gemm_bf16_tc(static_cast<const bf16*>(d_A), lda, static_cast<const bf16*>(d_W), M, N, K, ep,
                                e->tc_scratch(), static_cast<cudaStream_t>(cuda_stream));
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_gemm_bf16_ln");
  return SF_OK;
}

sf_status sf_attention_relpos(sf_engine* e, const void* d_qkv, const void* d_ptab, int R, const float* d_u,
                              const float* d_v, const int* h_seq_len, int n, void* d_ctx, int path,
                              void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_qkv || !d_ptab || !d_u || !d_v || !h_seq_len || !d_ctx) return fail(e, SF_EINVAL, "null pointer argument");
  if (e->cfg.precision != SF_BF16) return fail(e, SF_ESTATE, "sf_attention_relpos needs a bf16 engine");
  if (n < 1 || n > MAX_SEQ || (path != 0 && path != 1) || R < 1) return fail(e, SF_ESHAPE, "sequence count, path or R");
  if ((reinterpret_cast<uintptr_t>(d_qkv) | reinterpret_cast<uintptr_t>(d_ptab) | reinterpret_cast<uintptr_t>(d_ctx)) & 15)
    return fail(e, SF_EINVAL, "qkv, ptab and ctx must be 16-byte aligned");
  std::vector<int> lens(h_seq_len, h_seq_len + n);
  for (int v : lens)
    if (v < 1 || v > R) return fail(e, SF_ESHAPE, "sequence length must be in [1, R]");
  DescBlock* d = desc_begin(e);
  int M, tiles;
  fill_seq(d, lens, M, tiles);
  const int tiles2 = d->seq.tile2_off[n];
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = desc_upload(e, st);
  const bf16* qkv = static_cast<const bf16*>(d_qkv);
  const bf16* ptab = static_cast<const bf16*>(d_ptab);
  bf16* ctx = static_cast<bf16*>(d_ctx);
  if (ce == cudaSuccess)
    ce = path == 1 ? launch_relpos_attention_tc(qkv, ptab, R, d_u, d_v, ctx, &e->d_desc->seq, tiles2, M,
                                                *std::max_element(lens.begin(), lens.end()), e->tc_scratch(), st)
                   : launch_relpos_attention<bf16>(qkv, ptab, R, d_u, d_v, ctx, &e->d_desc->seq, tiles, M, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_attention_relpos");
  return SF_OK;
}

sf_status sf_attention_mha(sf_engine* e, const void* d_qkv, const int* h_seq_len, int n, void* d_ctx, int path,
                           void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_qkv || !h_seq_len || !d_ctx) return fail(e, SF_EINVAL, "null pointer argument");
  if (e->cfg.precision != SF_BF16) return fail(e, SF_ESTATE, "sf_attention_mha needs a bf16 engine");
  if (n < 1 || n > MAX_SEQ || path < 0 || path > 1) return fail(e, SF_ESHAPE, "sequence count or path");
  if ((reinterpret_cast<uintptr_t>(d_qkv) | reinterpret_cast<uintptr_t>(d_ctx)) & 15)
    return fail(e, SF_EINVAL, "qkv and ctx must be 16-byte aligned");
  std::vector<int> lens(h_seq_len, h_seq_len + n);
  for (int v : lens)
    if (v < 1 || v > e->max_seq_len) return fail(e, SF_ESHAPE, "sequence length out of range");
  DescBlock* d = desc_begin(e);
  int M, tiles;
  fill_seq(d, lens, M, tiles);
  const int tiles2 = d->seq.tile2_off[n];
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = desc_upload(e, st);
  const bf16* qkv = static_cast<const bf16*>(d_qkv);
  bf16* ctx = static_cast<bf16*>(d_ctx);
  if (ce == cudaSuccess)
    ce = path == 1   ? launch_mha_tc(qkv, ctx, &e->d_desc->seq, tiles2, M, *std::max_element(lens.begin(), lens.end()),
                                     e->d_err, st)
                     : launch_mha<bf16>(qkv, ctx, &e->d_desc->seq, tiles, M, e->max_seq_len, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_attention_mha");
  return SF_OK;
}

sf_status sf_default_seg_params(sf_seg_params* out) {
  if (!out) return SF_EINVAL;
  *out = sf_seg_params{0.5f, 0.5f, 0.0, 0.0, 0.0, 0.0};
  return SF_OK;
}

sf_status sf_segments(sf_engine* e, const float* d_probs, int stride_t, const int* h_n_frames, int n,
                      const sf_seg_params* prm, int max_seg, double* d_segs, int* d_counts, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_probs || !h_n_frames || !prm || !d_segs || !d_counts) return fail(e, SF_EINVAL, "null pointer argument");
  if (n < 1 || n > MAX_SEQ || stride_t < 1 || max_seg < 1) return fail(e, SF_ESHAPE, "n, stride_t or max_seg out of range");
  if (!(prm->onset >= prm->offset) || !(prm->offset >= 0.f) || !(prm->onset <= 1.f) || !(prm->pad_onset >= 0.0) ||
      !(prm->pad_offset >= 0.0) || !(prm->min_duration_on >= 0.0) || !(prm->min_duration_off >= 0.0))
    return fail(e, SF_EINVAL, "segment parameters: 0 <= offset <= onset <= 1, non-negative times");
  DescBlock* d = desc_begin(e);
  for (int i = 0; i < n; ++i) {
    if (h_n_frames[i] < 0 || h_n_frames[i] > stride_t) return fail(e, SF_ESHAPE, "n_frames out of [0, stride_t]");
    d->count[i] = h_n_frames[i];
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  SegArgs a{prm->onset, prm->offset, prm->pad_onset, prm->pad_offset, prm->min_duration_on, prm->min_duration_off,
            max_seg};
  cudaError_t ce = desc_upload(e, st);
  if (ce == cudaSuccess) ce = launch_segments(d_probs, stride_t, e->d_desc->count, n, a, d_segs, d_counts, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_segments");
  return SF_OK;
}

sf_status sf_set_option(sf_engine* e, int option, int value) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  switch (option) {
    case SF_OPT_GRAPHS: e->use_graphs = value != 0; break;
    case SF_OPT_PDL: e->use_pdl = value != 0; break;
    case SF_OPT_GEMM_PATH:
      if (value < 0 || value > 3) return fail(e, SF_EINVAL, "gemm path must be 0, 1, 2 or 3");
      e->gemm_path = value;
      break;
    case SF_OPT_ATTN_PATH:
      if (value != 0 && value != 1) return fail(e, SF_EINVAL, "attention path must be 0 or 1");
      e->attn_path = value;
      break;
    case SF_OPT_MEL_PATH:
      if (value != 0 && value != 1) return fail(e, SF_EINVAL, "front-end path must be 0 or 1");
      e->mel_path = value;
      break;
    case SF_OPT_SUB_PATH:
      if (value != 0 && value != 1) return fail(e, SF_EINVAL, "subsampling path must be 0 or 1");
      e->sub_path = value;
      break;
    case SF_OPT_LN_FUSE:
      if (value != 0 && value != 1) return fail(e, SF_EINVAL, "LayerNorm fusion must be 0 or 1");
      e->ln_fuse = value;
      break;
    case SF_OPT_TF_FUSE:
      if (value < 0 || value > 2) return fail(e, SF_EINVAL, "Transformer layer fusion must be 0, 1 or 2");
      e->tf_fuse = value;
      break;
    case SF_OPT_GEMM_PAIR_BN:
      if (value != 0 && value != 128 && value != 192 && value != 256)
        return fail(e, SF_EINVAL, "pair tile width must be 0, 128, 192 or 256");
      e->pair_bn = value;
      break;
    default: return fail(e, SF_EINVAL, "unknown option");
  }
  sf::g_launch_pdl = e->use_pdl;
  sf::g_gemm_pairs = e->gemm_path == 2 ? 2 : e->gemm_path == 3 ? 0 : 1;
  sf::g_gemm_pair_bn = e->pair_bn;
  return SF_OK;
}

sf_status sf_profile_enable(sf_engine* e, int enable) {
  if (!e) return SF_EINVAL;
  e->prof = enable != 0;
  e->prof_mask = enable == 1 ? 0xffffffffu : (uint32_t)enable >> 1;
  return SF_OK;
}

sf_status sf_profile_read(sf_engine* e, sf_kernel_stat* out, int max, int* n_out, int reset) {
  if (!e || !n_out || (max > 0 && !out)) return SF_EINVAL;
  double ms[K_COUNT] = {};
  for (int k = 0; k < K_COUNT; ++k) ms[k] = e->ms_acc[k];
  for (const ProfRec& r : e->recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      return fail(e, SF_ECUDA, "sf_profile_read: event query failed");
    ms[r.cls] += t;
  }
  int n = 0;
  for (int k = 0; k < K_COUNT; ++k) {
    if (e->launches[k] == 0) continue;
    if (n < max) {
      sf_kernel_stat& o = out[n];
      memset(&o, 0, sizeof(o));
      strncpy(o.name, KNAMES[k], sizeof(o.name) - 1);
      o.launches = e->launches[k];
      o.ms = ms[k];
      o.flops = e->kflops[k];
      o.bytes = e->kbytes[k];
    }
    ++n;
  }
  *n_out = n;
  if (reset) {
    for (int k = 0; k < K_COUNT; ++k) e->launches[k] = 0, e->kflops[k] = e->kbytes[k] = e->ms_acc[k] = 0;
    e->recs.clear();
    e->pool_used = 0;
  }
  return SF_OK;
}

sf_status sf_select_topk(sf_engine* e, const float* d_scores, const int* h_n, int n_sets, int stride, int k,
                         int* d_src, void* cuda_stream) {
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_scores || !h_n || !d_src) return fail(e, SF_EINVAL, "null pointer argument");
  if (n_sets < 1 || n_sets > MAX_SEQ || k < 1 || 4 * k > CAND_MAX || stride < 1)
    return fail(e, SF_ESHAPE, "set count, k or stride out of range");
  DescBlock* d = desc_begin(e);
  for (int i = 0; i < n_sets; ++i) {
    if (h_n[i] < 0 || h_n[i] > stride || h_n[i] > CAND_MAX) return fail(e, SF_ESHAPE, "candidate count out of range");
    d->n_cand[i] = h_n[i];
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = desc_upload(e, st);
  if (ce == cudaSuccess) {
    Scope sc(e, K_SELECT, 1, 0, 0, st);
    ce = launch_select_topk(d_scores, e->d_desc->n_cand, n_sets, stride, k, d_src, st);
  }
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_select_topk");
  return SF_OK;
}

}  // extern "C"

// ================================================================ streaming
namespace {

struct StepPlan {
  std::vector<int> sid, lc, n_new, cl, npop;
  std::vector<int64_t> m0, W;
};

void plan_sizes(const sf_stream* s, int id, int n_new, int& cl, int& npop) {
  cl = std::min(s->p.chunk_len, n_new);
  const int nF = s->n_f[id] + cl;
  npop = nF > s->p.fifo_len ? std::min(std::max(s->p.update_period, nF - s->p.fifo_len), nF) : 0;
}

void fill_step(sf_stream* s, DescBlock* d, const StepPlan& pl, int& M, int& tiles) {
  std::vector<int> lens;
  for (size_t i = 0; i < pl.sid.size(); ++i) {
    const int id = pl.sid[i];
    d->step.stream[i] = id;
    d->step.n_c[i] = s->n_c[id];
    d->step.n_f[i] = s->n_f[id];
    d->step.lc[i] = pl.lc[i];
    d->step.n_new[i] = pl.n_new[i];
    d->step.cl[i] = pl.cl[i];
    d->step.npop[i] = pl.npop[i];
    d->step.first_out[i] = s->n_c[id] + s->n_f[id];
    d->step.cur_c[i] = s->cur_c[id];
    d->step.cur_f[i] = s->cur_f[id];
    d->first[i] = s->n_c[id] + s->n_f[id];
    d->count[i] = pl.cl[i];
    d->dst[i] = id;
    lens.push_back(s->n_c[id] + s->n_f[id] + pl.n_new[i]);
  }
  fill_seq(d, lens, M, tiles);
  s->e->att_s2 = sum_sq(lens);
  s->e->att_tiles2 = d->seq.tile2_off[d->seq.n_seq];
  s->e->att_max_len = 0;
  for (int q_ = 0; q_ < d->seq.n_seq; ++q_)
    s->e->att_max_len = std::max(s->e->att_max_len, d->seq.off[q_ + 1] - d->seq.off[q_]);
}

// Host bookkeeping after a state update (sizes are data-independent).
void commit_sizes(sf_stream* s, const StepPlan& pl) {
  for (size_t i = 0; i < pl.sid.size(); ++i) {
    const int id = pl.sid[i];
    const int nF = s->n_f[id] + pl.cl[i];
    if (pl.npop[i] > 0) {
      s->n_f[id] = nF - pl.npop[i];
      s->cur_f[id] ^= 1;
      const int nC = s->n_c[id] + pl.npop[i];
      if (nC > s->p.spkcache_len) {
        s->n_c[id] = (s->p.spkcache_len / 4) * 4;
        s->cur_c[id] ^= 1;
      } else {
        s->n_c[id] = nC;
      }
    } else {
      s->n_f[id] = nF;
    }
    s->c0[id] += pl.cl[i];
  }
}

// Audio-in step inputs: stream buffers [n_streams][n_buf] (row = stream id,
// column 0 = absolute sample start[id], end[id] samples arrived) and each
// planned window's first mel frame m0[i].
struct AudioIn {
  const float* audio;
  int64_t n_buf;
  const int64_t* start;
  const int64_t* end;
  std::vector<int64_t> m0;
};

template <typename T>
cudaError_t stream_step_impl(sf_stream* s, const float* d_feats, int64_t t_buf, const StepPlan& pl,
                             float* d_chunk_probs, cudaStream_t st, const AudioIn* ain = nullptr) {
  sf_engine* e = s->e;
  DescBlock* d = desc_begin(e);
  const int n = (int)pl.sid.size();
  int64_t W_max = 0;
  for (int i = 0; i < n; ++i) {
    d->buf[i] = pl.sid[i];
    d->start[i] = pl.m0[i];
    d->frames[i] = pl.W[i];
    W_max = std::max(W_max, pl.W[i]);
  }
  if (ain) {   // audio-in step: the windows' features are computed from audio first
    for (int i = 0; i < n; ++i) {
      d->len[i] = ain->end[pl.sid[i]];
      d->win_f0[i] = ain->m0[i];
      d->win_a0[i] = ain->start[pl.sid[i]];
      d->win_nf[i] = (int)pl.W[i];
    }
    CK(ensure(e->mel, (size_t)s->n * 128 * W_max * 4));   // rows by stream id, as the pre-encode reads them
    CK(ensure(e->part, ((size_t)n * ((W_max + 31) / 32) * 128 * 4 + (size_t)n * 128 * 2) * 4));
    d_feats = static_cast<const float*>(e->mel.p);
    t_buf = W_max;
  }
  int M, tiles;
  fill_step(s, d, pl, M, tiles);
  const int T3 = (int)enc_frames(W_max);
  CK(ensure(e->emb, (size_t)n * T3 * e->cfg.d_model * sizeof(T)));
  CK(ensure_encode_ws(e, M));
  CK(prep_pre_encode(e, n, W_max, sizeof(T)));
  std::string key = stream_graph_prefix(s) + std::to_string(n) + "|" +
                    std::to_string(M) + "|" + std::to_string(tiles) + "|" + std::to_string(e->att_tiles2) + "|" +
                    std::to_string(W_max) + "|" +
                    std::to_string(t_buf) + "|" + std::to_string(reinterpret_cast<uintptr_t>(d_feats)) + "|" +
                    std::to_string(reinterpret_cast<uintptr_t>(d_chunk_probs));
  if (ain) key += "|a" + std::to_string(reinterpret_cast<uintptr_t>(ain->audio)) + "|" + std::to_string(ain->n_buf);
  return run_graph(e, key, st, [&](cudaStream_t st) -> cudaError_t {
    CK(desc_upload(e, st));
    if (n < s->n) CK(cudaMemsetAsync(d_chunk_probs, 0, (size_t)s->n * s->p.chunk_len * 4 * 4, st));
    if (ain) {
      MelArgs ma{e->d_desc->len};
      ma.f0 = e->d_desc->win_f0;
      ma.a0 = e->d_desc->win_a0;
      ma.nf = e->d_desc->win_nf;
      ma.row = e->d_desc->buf;
      RUN(K_MEL, e->mel_path ? 3 : 2, 0, (double)n * W_max * (160 * 4 + 128 * 4),
          launch_mel_windows(ain->audio, n, ain->n_buf, ma, e->d_mel_tab, static_cast<float*>(e->mel.p),
                             static_cast<float*>(e->part.p), (int)W_max, st, e->mel_path));
    }
    CK(run_pre_encode<T>(e, d_feats, t_buf, n, W_max, static_cast<T*>(e->emb.p), T3, st));
    RUN(K_ASSEMBLE, 1, 0, (double)M * e->cfg.d_model * (4 + sizeof(T)),
        launch_assemble<T>(static_cast<float*>(e->x.p), &e->d_desc->seq, &e->d_desc->step, s->sb,
                           static_cast<T*>(e->emb.p), T3, M, st));
    CK(run_encode<T>(e, M, tiles, static_cast<float*>(e->probs.p), st));
    RUN(K_EXTRACT, 1, 0, (double)n * s->p.chunk_len * 32,
        launch_extract_rows(static_cast<float*>(e->probs.p), &e->d_desc->seq, e->d_desc->first, e->d_desc->count,
                            e->d_desc->dst, n, d_chunk_probs, s->p.chunk_len, st));
    RUN(K_UPDATE, 1, 0, 0,
        launch_state_update<T>(static_cast<float*>(e->probs.p), &e->d_desc->seq, &e->d_desc->step, s->sb,
                               static_cast<T*>(e->emb.p), T3, n, nullptr, nullptr, nullptr, 0, st));
    return cudaSuccess;
  });
}

// Workspaces of a streaming step of n streams at its largest: window of
// 8 (1 + chunk_len + right_context) mel frames, encoder rows per stream up to
// the cache, the FIFO with a chunk, and the window's new frames.
cudaError_t reserve_stream_ws(sf_engine* e, int n, const sf_preset& p) {
  const size_t a = act_size(e);
  const int64_t W_max = 8 * (1 + (int64_t)p.chunk_len + p.right_context);
  const int64_t T3 = enc_frames(W_max);
  const int64_t S_max = (int64_t)p.spkcache_len + p.fifo_len + p.chunk_len + T3;
  g_ws_gen = &e->ws_gen;
  CK(ensure_encode_ws(e, (int)(n * S_max)));
  CK(ensure(e->emb, (size_t)n * T3 * e->cfg.d_model * a));
  CK(prep_pre_encode(e, n, W_max, a));
  CK(ensure(e->mel, (size_t)n * 128 * W_max * 4));
  CK(ensure(e->part, ((size_t)n * ((W_max + 31) / 32) * 128 * 4 + (size_t)n * 128 * 2) * 4));
  return cudaSuccess;
}

}  // namespace

extern "C" {

sf_status sf_stream_create(sf_engine* e, const sf_preset* p, int n_streams, sf_stream** out) {
  if (check_engine(e) != SF_OK || !p || !out) return SF_EINVAL;
  *out = nullptr;
  if (n_streams < 1 || n_streams > std::min(MAX_SEQ, e->cfg.max_batch)) return fail(e, SF_ESHAPE, "n_streams out of range");
  if (p->chunk_len < 1 || p->right_context < 0 || p->fifo_len < 0 || p->update_period < 1 || p->spkcache_len < 4 ||
      p->spkcache_len > e->cfg.spkcache_len || p->spkcache_len % 4)
    return fail(e, SF_EINVAL, "invalid preset");
  const int win = p->spkcache_len + p->fifo_len + p->chunk_len + p->right_context;
  if (win > e->max_seq_len) return fail(e, SF_ESHAPE, "preset window longer than the position table");
  if (p->spkcache_len + p->fifo_len + p->chunk_len > CAND_MAX) return fail(e, SF_ESHAPE, "preset too large for compression");
  std::unique_ptr<sf_stream> s(new sf_stream());
  s->e = e;
  s->serial = ++e->stream_serial;
  s->p = *p;
  s->n = n_streams;
  const int D = e->cfg.d_model;
  const size_t a = act_size(e);
  StateBufs& sb = s->sb;
  sb.cap_c = p->spkcache_len;
  sb.cap_f = p->fifo_len + p->chunk_len;
  sb.D = D;
  sb.cache_len = p->spkcache_len;
  const size_t ce_b = (size_t)n_streams * sb.cap_c * D * a, cp_b = (size_t)n_streams * sb.cap_c * 16;
  const size_t fe_b = (size_t)n_streams * sb.cap_f * D * a, fp_b = (size_t)n_streams * sb.cap_f * 16;
  const size_t sm_b = (size_t)n_streams * D * 4, sc_b = (size_t)n_streams * 4;
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  const size_t total = 2 * (al(ce_b) + al(cp_b) + al(fe_b) + al(fp_b)) + al(sm_b) + al(sc_b);
  if (cudaMalloc(&s->alloc, total) != cudaSuccess) return fail(e, SF_ENOMEM, "stream state");
  uint8_t* q = static_cast<uint8_t*>(s->alloc);
  for (int k = 0; k < 2; ++k) {
    sb.cache_emb[k] = q; q += al(ce_b);
    sb.cache_preds[k] = reinterpret_cast<float*>(q); q += al(cp_b);
    sb.fifo_emb[k] = q; q += al(fe_b);
    sb.fifo_preds[k] = reinterpret_cast<float*>(q); q += al(fp_b);
  }
  sb.sil_mean = reinterpret_cast<float*>(q); q += al(sm_b);
  sb.sil_count = reinterpret_cast<int*>(q);
  s->n_c.assign(n_streams, 0);
  s->n_f.assign(n_streams, 0);
  s->cur_c.assign(n_streams, 0);
  s->cur_f.assign(n_streams, 0);
  s->finished.assign(n_streams, 0);
  s->c0.assign(n_streams, 0);
  if (cudaMemset(s->alloc, 0, total) != cudaSuccess) {
    cudaFree(s->alloc);
    return fail(e, SF_ECUDA, "stream state init");
  }
  // The engine's workspaces at this preset's largest step, reserved now: a
  // buffer that grew during the steps would move and invalidate every step
  // graph captured before it.
  if (reserve_stream_ws(e, n_streams, *p) != cudaSuccess) {
    cudaFree(s->alloc);
    return fail(e, SF_ENOMEM, "stream workspaces");
  }
  e->streams.push_back(s.get());
  *out = s.release();
  return SF_OK;
}

sf_status sf_stream_destroy(sf_stream* s) {
  if (!s) return SF_EINVAL;
  cudaDeviceSynchronize();
  if (s->e) {
    destroy_graphs_with_prefix(s->e, stream_graph_prefix(s));   // they hold this stream's buffers
    auto& v = s->e->streams;
    v.erase(std::remove(v.begin(), v.end(), s), v.end());
  }
  if (s->alloc) cudaFree(s->alloc);
  delete s;
  return SF_OK;
}

sf_status sf_stream_reset(sf_stream* s, const int* ids, int n) {
  if (!s) return SF_EINVAL;
  if (ids && n < 0) return fail(s->e, SF_EINVAL, "negative id count");
  std::vector<int> list;
  if (ids) list.assign(ids, ids + n);
  else for (int i = 0; i < s->n; ++i) list.push_back(i);
  for (int id : list)
    if (id < 0 || id >= s->n) return fail(s->e, SF_EINVAL, "stream id out of range");
  // A step still running on any caller stream reads and writes the silence
  // statistics: wait for it, clear them, and wait for the clear, so that the
  // next step (on any stream) starts from the cleared state.
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(s->e, SF_ECUDA, "reset: device");
  for (int id : list) {
    s->n_c[id] = s->n_f[id] = 0;
    s->cur_c[id] = s->cur_f[id] = 0;
    s->finished[id] = 0;
    s->c0[id] = 0;
    // the silence mean restarts from zero; cache/FIFO contents are dead once sizes are 0
    if (cudaMemset(s->sb.sil_mean + (size_t)id * s->sb.D, 0, (size_t)s->sb.D * 4) != cudaSuccess ||
        cudaMemset(s->sb.sil_count + id, 0, sizeof(int)) != cudaSuccess)
      return fail(s->e, SF_ECUDA, "reset: clear");
  }
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(s->e, SF_ECUDA, "reset: device");
  return SF_OK;
}

sf_status sf_stream_window(const sf_stream* s, int id, int64_t total, int64_t* h_start, int64_t* h_end) {
  if (!s || !h_start || !h_end || id < 0 || id >= s->n) return SF_EINVAL;
  const int64_t c0 = s->c0[id];
  const int lc = c0 > 0 ? 1 : 0;
  *h_start = 8 * (c0 - lc);
  *h_end = std::min<int64_t>(8 * (c0 + s->p.chunk_len + s->p.right_context), total);
  return SF_OK;
}

sf_status sf_stream_step(sf_stream* s, const float* d_feats, int64_t t_buf, const int64_t* h_feat_start,
                         const int64_t* h_feat_end, float* d_chunk_probs, int* h_n_out, void* cuda_stream) {
  if (!s) return SF_EINVAL;
  sf_engine* e = s->e;
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_feats || !h_feat_start || !h_feat_end || !d_chunk_probs) return fail(e, SF_EINVAL, "null pointer argument");
  StepPlan pl;
  for (int id = 0; id < s->n; ++id) {
    if (s->finished[id]) continue;
    const int64_t c0 = s->c0[id];
    const int lc = c0 > 0 ? 1 : 0;
    const int64_t m0 = 8 * (c0 - lc);
    const int64_t m1 = std::min<int64_t>(8 * (c0 + s->p.chunk_len + s->p.right_context), h_feat_end[id]);
    if (m1 <= 8 * c0) return fail(e, SF_ESTATE, "stream " + std::to_string(id) + " has no frames left");
    if (m0 < h_feat_start[id] || m1 - h_feat_start[id] > t_buf)
      return fail(e, SF_ESHAPE, "stream " + std::to_string(id) + ": window outside the feature buffer");
    const int64_t W = m1 - m0;
    const int n_new = (int)(enc_frames(W) - lc);
    int cl, npop;
    plan_sizes(s, id, n_new, cl, npop);
    pl.sid.push_back(id);
    pl.lc.push_back(lc);
    pl.n_new.push_back(n_new);
    pl.cl.push_back(cl);
    pl.npop.push_back(npop);
    pl.m0.push_back(m0 - h_feat_start[id]);
    pl.W.push_back(W);
  }
  if (pl.sid.empty()) return fail(e, SF_ESTATE, "all streams finished");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = e->cfg.precision == SF_BF16 ? stream_step_impl<bf16>(s, d_feats, t_buf, pl, d_chunk_probs, st)
                                               : stream_step_impl<float>(s, d_feats, t_buf, pl, d_chunk_probs, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_stream_step");
  if (h_n_out)
    for (int id = 0; id < s->n; ++id) h_n_out[id] = 0;
  for (size_t i = 0; i < pl.sid.size(); ++i) {
    const int id = pl.sid[i];
    if (h_n_out) h_n_out[id] = pl.cl[i];
    const int64_t end_frame = enc_frames(h_feat_end[id]);
    if (s->c0[id] + pl.cl[i] >= end_frame) s->finished[id] = 1;
  }
  commit_sizes(s, pl);
  return SF_OK;
}

sf_status sf_stream_update(sf_stream* s, const float* d_preds, const void* d_new_embs, int64_t new_stride,
                           const int* h_n_new, float* d_scores, int* d_src, const float* d_scores_in,
                           void* cuda_stream) {
  if (!s) return SF_EINVAL;
  sf_engine* e = s->e;
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_preds || !d_new_embs || !h_n_new) return fail(e, SF_EINVAL, "null pointer argument");
  StepPlan pl;
  for (int id = 0; id < s->n; ++id) {
    if (h_n_new[id] <= 0) continue;
    if (h_n_new[id] > new_stride) return fail(e, SF_ESHAPE, "n_new larger than new_stride");
    if (s->finished[id]) return fail(e, SF_ESTATE, "stream finished");
    int cl, npop;
    plan_sizes(s, id, h_n_new[id], cl, npop);
    pl.sid.push_back(id);
    pl.lc.push_back(0);
    pl.n_new.push_back(h_n_new[id]);
    pl.cl.push_back(cl);
    pl.npop.push_back(npop);
    pl.m0.push_back(0);
    pl.W.push_back(0);
  }
  if (pl.sid.empty()) return SF_OK;
  DescBlock* d = desc_begin(e);
  int M, tiles;
  fill_step(s, d, pl, M, tiles);
  // the embeddings buffer is indexed by sequence: pass the rows of each listed stream
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const size_t a = act_size(e);
  const int D = e->cfg.d_model;
  const int n = (int)pl.sid.size();
  cudaError_t ce = ensure(e->emb, (size_t)n * new_stride * D * a);
  for (int i = 0; i < n && ce == cudaSuccess; ++i)
    ce = cudaMemcpyAsync(static_cast<uint8_t*>(e->emb.p) + (size_t)i * new_stride * D * a,
                         static_cast<const uint8_t*>(d_new_embs) + (size_t)pl.sid[i] * new_stride * D * a,
                         (size_t)new_stride * D * a, cudaMemcpyDeviceToDevice, st);
  if (ce == cudaSuccess) ce = desc_upload(e, st);
  const int score_stride = s->p.spkcache_len + s->p.fifo_len + s->p.chunk_len;
  Scope sc(e, K_UPDATE, ce == cudaSuccess ? 1 : 0, 0, 0, st);
  if (ce == cudaSuccess)
    ce = e->cfg.precision == SF_BF16
             ? launch_state_update<bf16>(d_preds, &e->d_desc->seq, &e->d_desc->step, s->sb, static_cast<bf16*>(e->emb.p),
                                         (int)new_stride, n, d_scores, d_src, d_scores_in, score_stride, st)
             : launch_state_update<float>(d_preds, &e->d_desc->seq, &e->d_desc->step, s->sb,
                                          static_cast<float*>(e->emb.p), (int)new_stride, n, d_scores, d_src,
                                          d_scores_in, score_stride, st);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_stream_update");
  commit_sizes(s, pl);
  return SF_OK;
}

sf_status sf_stream_step_audio(sf_stream* s, const float* d_audio, int64_t n_buf, const int64_t* h_audio_start,
                               const int64_t* h_audio_end, const int* h_final, float* d_chunk_probs, int* h_n_out,
                               void* cuda_stream) {
  if (!s) return SF_EINVAL;
  sf_engine* e = s->e;
  if (check_engine(e) != SF_OK) return SF_EINVAL;
  if (!d_audio || !h_audio_start || !h_audio_end || !h_final || !d_chunk_probs)
    return fail(e, SF_EINVAL, "null pointer argument");
  if (n_buf < 1) return fail(e, SF_ESHAPE, "n_buf must be positive");
  StepPlan pl;
  AudioIn ain{d_audio, n_buf, h_audio_start, h_audio_end, {}};
  for (int id = 0; id < s->n; ++id) {
    if (s->finished[id]) continue;
    const int64_t a0 = h_audio_start[id], end = h_audio_end[id];
    if (a0 < 0 || end < a0 || end - a0 > n_buf)
      return fail(e, SF_ESHAPE, "stream " + std::to_string(id) + ": audio range outside its buffer row");
    const int64_t c0 = s->c0[id];
    const int lc = c0 > 0 ? 1 : 0;
    const int64_t m0 = 8 * (c0 - lc);
    const int64_t need = 8 * (c0 + s->p.chunk_len + s->p.right_context);   // mel frames of chunk + look-ahead
    const int64_t m1 = std::min<int64_t>(need, end / 160);
    // a window is ready once its last frame's samples have arrived (last
    // frame centred at 160 (need - 1), reaching 256 samples past it), or at
    // the end of the stream's audio
    const bool ready = h_final[id] ? m1 > 8 * c0 : end >= 160 * need + 96;
    if (!ready) continue;
    if (a0 > std::max<int64_t>(0, 160 * m0 - 257))
      return fail(e, SF_ESHAPE, "stream " + std::to_string(id) + ": buffer starts after the window's first samples");
    const int64_t W = m1 - m0;
    const int n_new = (int)(enc_frames(W) - lc);
    int cl, npop;
    plan_sizes(s, id, n_new, cl, npop);
    pl.sid.push_back(id);
    pl.lc.push_back(lc);
    pl.n_new.push_back(n_new);
    pl.cl.push_back(cl);
    pl.npop.push_back(npop);
    pl.m0.push_back(0);   // window-local features
    pl.W.push_back(W);
    ain.m0.push_back(m0);
  }
  if (h_n_out)
    for (int id = 0; id < s->n; ++id) h_n_out[id] = 0;
  if (pl.sid.empty()) return SF_OK;   // no stream has a full window yet
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = e->cfg.precision == SF_BF16 ? stream_step_impl<bf16>(s, nullptr, 0, pl, d_chunk_probs, st, &ain)
                                               : stream_step_impl<float>(s, nullptr, 0, pl, d_chunk_probs, st, &ain);
  if (ce != cudaSuccess) return cuda_fail(e, ce, "sf_stream_step_audio");
  for (size_t i = 0; i < pl.sid.size(); ++i) {
    const int id = pl.sid[i];
    if (h_n_out) h_n_out[id] = pl.cl[i];
    if (h_final[id] && s->c0[id] + pl.cl[i] >= enc_frames(h_audio_end[id] / 160)) s->finished[id] = 1;
  }
  commit_sizes(s, pl);
  return SF_OK;
}

sf_status sf_stream_get_state(sf_stream* s, int id, sf_state_view* v, void* cuda_stream) {
  if (!s || !v || id < 0 || id >= s->n || !s->e) return SF_EINVAL;
  sf_engine* e = s->e;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const size_t a = act_size(e);
  const int D = s->sb.D;
  v->n_cache = s->n_c[id];
  v->n_fifo = s->n_f[id];
  v->next_frame = s->c0[id];
  v->finished = s->finished[id];
  const uint8_t* ce_ = static_cast<const uint8_t*>(s->sb.cache_emb[s->cur_c[id]]) + (size_t)id * s->sb.cap_c * D * a;
  const float* cp = s->sb.cache_preds[s->cur_c[id]] + (size_t)id * s->sb.cap_c * 4;
  const uint8_t* fe = static_cast<const uint8_t*>(s->sb.fifo_emb[s->cur_f[id]]) + (size_t)id * s->sb.cap_f * D * a;
  const float* fp = s->sb.fifo_preds[s->cur_f[id]] + (size_t)id * s->sb.cap_f * 4;
  cudaError_t c = cudaSuccess;
  if (v->d_cache_emb && v->n_cache) c = cudaMemcpyAsync(v->d_cache_emb, ce_, (size_t)v->n_cache * D * a, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->d_cache_preds && v->n_cache) c = cudaMemcpyAsync(v->d_cache_preds, cp, (size_t)v->n_cache * 16, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->d_fifo_emb && v->n_fifo) c = cudaMemcpyAsync(v->d_fifo_emb, fe, (size_t)v->n_fifo * D * a, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->d_fifo_preds && v->n_fifo) c = cudaMemcpyAsync(v->d_fifo_preds, fp, (size_t)v->n_fifo * 16, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->d_sil_mean) c = cudaMemcpyAsync(v->d_sil_mean, s->sb.sil_mean + (size_t)id * D, (size_t)D * 4, cudaMemcpyDeviceToDevice, st);
  int cnt = 0;
  if (c == cudaSuccess) c = cudaMemcpyAsync(&cnt, s->sb.sil_count + id, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (c == cudaSuccess) c = cudaStreamSynchronize(st);
  if (c != cudaSuccess) return cuda_fail(e, c, "sf_stream_get_state");
  v->sil_count = cnt;
  return SF_OK;
}

sf_status sf_stream_set_state(sf_stream* s, int id, const sf_state_view* v, void* cuda_stream) {
  if (!s || !v || id < 0 || id >= s->n || !s->e) return SF_EINVAL;
  sf_engine* e = s->e;
  if (v->n_cache < 0 || v->n_cache > s->sb.cap_c || v->n_fifo < 0 || v->n_fifo > s->p.fifo_len || v->next_frame < 0 ||
      v->sil_count < 0)
    return fail(e, SF_ESHAPE, "state sizes out of range");
  if ((v->n_cache && (!v->d_cache_emb || !v->d_cache_preds)) || (v->n_fifo && (!v->d_fifo_emb || !v->d_fifo_preds)) ||
      !v->d_sil_mean)
    return fail(e, SF_EINVAL, "null state buffer");
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  const size_t a = act_size(e);
  const int D = s->sb.D;
  s->cur_c[id] = s->cur_f[id] = 0;
  uint8_t* ce_ = static_cast<uint8_t*>(s->sb.cache_emb[0]) + (size_t)id * s->sb.cap_c * D * a;
  float* cp = s->sb.cache_preds[0] + (size_t)id * s->sb.cap_c * 4;
  uint8_t* fe = static_cast<uint8_t*>(s->sb.fifo_emb[0]) + (size_t)id * s->sb.cap_f * D * a;
  float* fp = s->sb.fifo_preds[0] + (size_t)id * s->sb.cap_f * 4;
  cudaError_t c = cudaSuccess;
  if (v->n_cache) c = cudaMemcpyAsync(ce_, v->d_cache_emb, (size_t)v->n_cache * D * a, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->n_cache) c = cudaMemcpyAsync(cp, v->d_cache_preds, (size_t)v->n_cache * 16, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->n_fifo) c = cudaMemcpyAsync(fe, v->d_fifo_emb, (size_t)v->n_fifo * D * a, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess && v->n_fifo) c = cudaMemcpyAsync(fp, v->d_fifo_preds, (size_t)v->n_fifo * 16, cudaMemcpyDeviceToDevice, st);
  if (c == cudaSuccess) c = cudaMemcpyAsync(s->sb.sil_mean + (size_t)id * D, v->d_sil_mean, (size_t)D * 4, cudaMemcpyDeviceToDevice, st);
  const int cnt = v->sil_count;
  if (c == cudaSuccess) c = cudaMemcpyAsync(s->sb.sil_count + id, &cnt, sizeof(int), cudaMemcpyHostToDevice, st);
  if (c == cudaSuccess) c = cudaStreamSynchronize(st);
  if (c != cudaSuccess) return cuda_fail(e, c, "sf_stream_set_state");
  s->n_c[id] = v->n_cache;
  s->n_f[id] = v->n_fifo;
  s->c0[id] = v->next_frame;
  s->finished[id] = v->finished;
  return SF_OK;
}

}  // extern "C"
