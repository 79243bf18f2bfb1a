// Offline forward of the Nemotron-3 diarization variant ("Enable
// Nemotron-3-Diarization on MLX, CUDA, XNNPACK, and Vulkan", model
// description: 16 kHz mono audio, 128-bin mel features stacked to an 80 ms
// encoder frame rate, a 31-layer Transformer with rotary position embedding,
// a Conv1D upsampling head giving the activity of up to 8 speakers every
// 10 ms; Transformers "Nemotron 3 Diarization": logits (1, frames, 8), one
// frame every 10 ms, positions restarting at 0 for each window).
//
// Readings where the pages are silent (the same ones the CPU oracle states):
// d_model 512 in 8 heads of 64 and FFN 2048 (about 98M parameters with 31
// layers); frame-major stacking of 8 normalised mel frames (the engine's
// front-end) into 1024 features and a Linear 1024 -> 512; pre-LN layers
// (x += MHA(LN1(x)), x += FFN(LN2(x)), swish FFN) and a final LayerNorm;
// rotate-half RoPE on queries and keys with positions from each clip's
// start; a transposed 1-D convolution with kernel = stride = 8 as the head
// (one 512 -> 8 frames x 8 speakers map per encoder frame) and a sigmoid.
//
// Pipeline (bf16 operands, fp32 accumulation and residual stream): log-mel
// (the engine's front-end kernels), stacking, then per layer the tcgen05
// Q|K|V projection, RoPE in place, the tcgen05 attention (heads of 64), the
// output projection with the residual and LN2 in its epilogue, the swish FFN
// up-projection and the down-projection with the residual and the next
// layer's LN1 (or the final LN) in its epilogue; the head as a GEMM whose 64
// output columns per encoder frame are its 8 output frames x 8 speakers.
#include <algorithm>
#include <memory>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/sf.h"
#include "blob.h"
#include "common.cuh"
#include "frontend.h"
#include "layers.h"

namespace sf {
namespace {

constexpr int NM_D = 512, NM_H = 8, NM_HD = 64, NM_FF = 2048, NM_SPK = 8, NM_UP = 8, NM_STACK = 8, NM_MELS = 128;
constexpr int NM_IN = NM_STACK * NM_MELS;   // 1024 stacked features

// Encoder frame r of clip s (rows packed clip after clip) <- mel frames
// 8t .. 8t+7 of the clip's channels-first features, frame-major (column
// k * 128 + f); frames at or past the clip's L are zero.
__global__ void __launch_bounds__(256) nem_stack_kernel(const float* __restrict__ mel, int64_t T_cols,
                                                        const int64_t* __restrict__ len, const SeqTable* __restrict__ seq,
                                                        bf16* __restrict__ out) {
  SF_PDL_ENTRY();
  const int r = blockIdx.x;
  const int s = seq_of_row(seq, r);
  const int t = r - seq->off[s];
  const int64_t L = len[s] / 160;
  const float* src = mel + (int64_t)s * NM_MELS * T_cols;
  for (int c = threadIdx.x; c < NM_IN; c += blockDim.x) {
    const int k = c / NM_MELS, f = c % NM_MELS;
    const int64_t fr = 8 * (int64_t)t + k;
    out[(int64_t)r * NM_IN + c] = __float2bfloat16_rn(fr < L ? src[(int64_t)f * T_cols + fr] : 0.f);
  }
}

// Rotary embedding in place on the query and key columns of qkv [M x 1536]
// (one warp per row): in head h, dims i and i + 32 rotate by the angle
// p * 10000^(-2i/64), p the row's position in its clip.
__global__ void __launch_bounds__(256) nem_rope_kernel(bf16* __restrict__ qkv, const SeqTable* __restrict__ seq, int M) {
  SF_PDL_ENTRY();
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int i = threadIdx.x & 31;
  if (r >= M) return;
  const int p = r - seq->off[seq_of_row(seq, r)];
  const float inv = powf(10000.f, -2.f * (float)i / (float)NM_HD);
  float sn, cs;
  sincosf((float)p * inv, &sn, &cs);
  bf16* row = qkv + (int64_t)r * 3 * NM_D;
#pragma unroll
  for (int part = 0; part < 2; ++part) {
#pragma unroll
    for (int h = 0; h < NM_H; ++h) {
      bf16* x = row + part * NM_D + h * NM_HD;
      const float a = __bfloat162float(x[i]), b = __bfloat162float(x[i + NM_HD / 2]);
      x[i] = __float2bfloat16_rn(a * cs - b * sn);
      x[i + NM_HD / 2] = __float2bfloat16_rn(b * cs + a * sn);
    }
  }
}

// Head: logits [M x 64] (column k * 8 + s = output frame 8t + k of speaker s
// for encoder frame t) -> probs [B][L_max][8] = sigmoid, frames < L only.
__global__ void __launch_bounds__(256) nem_head_out_kernel(const float* __restrict__ logits,
                                                           const int64_t* __restrict__ len,
                                                           const SeqTable* __restrict__ seq, int M, int64_t L_max,
                                                           float* __restrict__ probs) {
  SF_PDL_ENTRY();
  const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (g >= (int64_t)M * NM_UP * NM_SPK) return;
  const int r = (int)(g / (NM_UP * NM_SPK)), c = (int)(g % (NM_UP * NM_SPK));
  const int s = seq_of_row(seq, r);
  const int t = r - seq->off[s];
  const int64_t fr = (int64_t)NM_UP * t + c / NM_SPK;
  if (fr < len[s] / 160) probs[((int64_t)s * L_max + fr) * NM_SPK + c % NM_SPK] = 1.f / (1.f + expf(-logits[g]));
}

struct NemLayer {
  bf16 *wqkv, *wo, *w1, *w2;
  float *bqkv, *bo, *ln1_g, *ln1_b, *ln2_g, *ln2_b, *b1, *b2;
};

}  // namespace
}  // namespace sf

using namespace sf;

struct sf_nem_engine {
  int device = 0;
  sf_nem_config cfg{};
  std::string err;
  void* d_weights = nullptr;
  bf16* stack_w = nullptr;
  float* stack_b = nullptr;
  std::vector<NemLayer> layers;
  float *fln_g = nullptr, *fln_b = nullptr;
  bf16* head_w = nullptr;   // [64 x 512]: row k * 8 + s
  float* head_b = nullptr;
  MelTables* d_mel_tab = nullptr;
  void* d_ws = nullptr;     // workspace (one allocation, carved below)
  float *mel = nullptr, *part = nullptr, *x = nullptr, *logits = nullptr;
  bf16 *stk = nullptr, *h = nullptr, *big = nullptr, *ctx = nullptr;
  int64_t* d_len = nullptr;
  SeqTable* d_seq = nullptr;
  SeqTable* h_seq = nullptr;   // pinned host copy of the sequence table
  int* d_err = nullptr;
  int64_t M_max = 0;
};

namespace {

sf_status nem_fail(sf_nem_engine* e, sf_status s, const std::string& m) {
  if (e) e->err = m;
  return s;
}

// x (f32 [M x 512]) += alpha (A W^T + b); h <- act(LN(x)) with (g, b): in
// the projection's epilogue where the row blocks' clusters fit one wave,
// else as a projection and a LayerNorm kernel.
cudaError_t nem_resid_ln(sf_nem_engine* e, const bf16* A, int lda, const bf16* W, int M, int K, const float* bias,
                         float* x, const float* g, const float* b, bf16* h, cudaStream_t st) {
  const TcScratch sc{e->d_err, nullptr, 0, nullptr, 0};
  Epi ep{};
  ep.bias = bias;
  ep.out = x;
  ep.ldo = NM_D;
  ep.alpha = 1.f;
  if (gemm_ln_fusable(M, NM_D, K)) {
    ep.kind = EPI_RESID_LN;
    ep.ln_g = g;
    ep.ln_b = b;
    ep.ln_h = h;
    ep.ldh = NM_D;
    ep.ln_xnorm = 0;
    return gemm_bf16_tc(A, lda, W, M, NM_D, K, ep, sc, st);
  }
  ep.kind = EPI_RESID;
  cudaError_t r = gemm_bf16_tc(A, lda, W, M, NM_D, K, ep, sc, st);
  if (r != cudaSuccess) return r;
  return launch_layernorm<bf16>(x, g, b, M, NM_D, false, h, st);
}

cudaError_t nem_gemm(sf_nem_engine* e, const bf16* A, int lda, const bf16* W, int M, int N, int K, int kind,
                     const float* bias, void* out, int ldo, cudaStream_t st) {
  const TcScratch sc{e->d_err, nullptr, 0, nullptr, 0};
  Epi ep{};
  ep.kind = kind;
  ep.bias = bias;
  ep.out = out;
  ep.ldo = ldo;
  ep.alpha = 1.f;
  return gemm_bf16_tc(A, lda, W, M, N, K, ep, sc, st);
}

}  // namespace

extern "C" {

sf_status sf_nem_default_config(sf_nem_config* c) {
  if (!c) return SF_EINVAL;
  c->n_layers = 31;
  c->d_model = NM_D;
  c->ff = NM_FF;
  c->n_spk = NM_SPK;
  c->max_batch = 1;
  c->max_samples = 1920000;
  return SF_OK;
}

sf_status sf_nem_create(const void* h_blob, uint64_t nbytes, const sf_nem_config* cfg, sf_nem_engine** out) {
  if (!h_blob || !cfg || !out) return SF_EINVAL;
  *out = nullptr;
  if (cfg->d_model != NM_D || cfg->ff != NM_FF || cfg->n_spk != NM_SPK || cfg->n_layers < 1 || cfg->n_layers > 64 ||
      cfg->max_batch < 1 || cfg->max_batch > MAX_SEQ || cfg->max_samples < 1600 || cfg->max_samples > 230400000LL)
    return SF_EINVAL;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
                                                cudaSuccess || major != 10)
    return SF_EDEVICE;
  auto e = std::make_unique<sf_nem_engine>();
  e->device = dev;
  e->cfg = *cfg;
  std::unordered_map<std::string, TensorRef> m;
  std::string perr;
  if (!parse_blob(h_blob, nbytes, m, perr)) return SF_EFORMAT;
  auto get = [&](const std::string& n, std::vector<uint32_t> shape) -> const float* {
    auto it = m.find(n);
    if (it == m.end() || it->second.shape != shape) return nullptr;
    return it->second.data;
  };
  // host staging of all weights, then one upload
  std::vector<uint8_t> host;
  std::vector<std::pair<void**, size_t>> fix;
  auto add = [&](void** slot, const void* src, size_t bytes) {
    const size_t off = (host.size() + 255) & ~size_t(255);
    host.resize(off + bytes);
    memcpy(host.data() + off, src, bytes);
    fix.push_back({slot, off});
  };
  auto add_bf16 = [&](bf16** slot, const std::vector<float>& v) {
    std::vector<uint16_t> b(v.size());
    for (size_t i = 0; i < v.size(); ++i) b[i] = f2bf_bits(v[i]);
    add(reinterpret_cast<void**>(slot), b.data(), b.size() * 2);
  };
  auto vec = [](const float* p, size_t n) { return std::vector<float>(p, p + n); };
  const int L = cfg->n_layers;
  e->layers.resize(L);
  const float* sw = get("nem.stack.weight", {NM_D, NM_IN});
  const float* sb = get("nem.stack.bias", {NM_D});
  if (!sw || !sb) return SF_EFORMAT;
  add_bf16(&e->stack_w, vec(sw, (size_t)NM_D * NM_IN));
  add(reinterpret_cast<void**>(&e->stack_b), sb, NM_D * 4);
  for (int l = 0; l < L; ++l) {
    const std::string p = "nem.layers." + std::to_string(l) + ".";
    NemLayer& w = e->layers[l];
    std::vector<float> wqkv, bqkv;
    for (const char* q : {"q", "k", "v"}) {
      const float* a = get(p + "att." + q + ".weight", {NM_D, NM_D});
      const float* b = get(p + "att." + q + ".bias", {NM_D});
      if (!a || !b) return SF_EFORMAT;
      wqkv.insert(wqkv.end(), a, a + (size_t)NM_D * NM_D);
      bqkv.insert(bqkv.end(), b, b + NM_D);
    }
    add_bf16(&w.wqkv, wqkv);
    add(reinterpret_cast<void**>(&w.bqkv), bqkv.data(), bqkv.size() * 4);
    const float *wo = get(p + "att.o.weight", {NM_D, NM_D}), *bo = get(p + "att.o.bias", {NM_D});
    const float *g1 = get(p + "ln1.weight", {NM_D}), *be1 = get(p + "ln1.bias", {NM_D});
    const float *g2 = get(p + "ln2.weight", {NM_D}), *be2 = get(p + "ln2.bias", {NM_D});
    const float *w1 = get(p + "ff.linear1.weight", {NM_FF, NM_D}), *b1 = get(p + "ff.linear1.bias", {NM_FF});
    const float *w2 = get(p + "ff.linear2.weight", {NM_D, NM_FF}), *b2 = get(p + "ff.linear2.bias", {NM_D});
    if (!wo || !bo || !g1 || !be1 || !g2 || !be2 || !w1 || !b1 || !w2 || !b2) return SF_EFORMAT;
    add_bf16(&w.wo, vec(wo, (size_t)NM_D * NM_D));
    add(reinterpret_cast<void**>(&w.bo), bo, NM_D * 4);
    add(reinterpret_cast<void**>(&w.ln1_g), g1, NM_D * 4);
    add(reinterpret_cast<void**>(&w.ln1_b), be1, NM_D * 4);
    add(reinterpret_cast<void**>(&w.ln2_g), g2, NM_D * 4);
    add(reinterpret_cast<void**>(&w.ln2_b), be2, NM_D * 4);
    add_bf16(&w.w1, vec(w1, (size_t)NM_FF * NM_D));
    add(reinterpret_cast<void**>(&w.b1), b1, NM_FF * 4);
    add_bf16(&w.w2, vec(w2, (size_t)NM_D * NM_FF));
    add(reinterpret_cast<void**>(&w.b2), b2, NM_D * 4);
  }
  const float *fg = get("nem.final_ln.weight", {NM_D}), *fb = get("nem.final_ln.bias", {NM_D});
  const float *hw = get("nem.head.weight", {NM_D, NM_SPK, NM_UP}), *hb = get("nem.head.bias", {NM_SPK});
  if (!fg || !fb || !hw || !hb) return SF_EFORMAT;
  add(reinterpret_cast<void**>(&e->fln_g), fg, NM_D * 4);
  add(reinterpret_cast<void**>(&e->fln_b), fb, NM_D * 4);
  {   // transposed-conv weight [c][s][k] -> GEMM rows k * 8 + s, bias per row
    std::vector<float> hg((size_t)NM_UP * NM_SPK * NM_D), hbg(NM_UP * NM_SPK);
    for (int k = 0; k < NM_UP; ++k)
      for (int s = 0; s < NM_SPK; ++s) {
        for (int c = 0; c < NM_D; ++c) hg[(size_t)(k * NM_SPK + s) * NM_D + c] = hw[((size_t)c * NM_SPK + s) * NM_UP + k];
        hbg[k * NM_SPK + s] = hb[s];
      }
    add_bf16(&e->head_w, hg);
    add(reinterpret_cast<void**>(&e->head_b), hbg.data(), hbg.size() * 4);
  }
  if (cudaMalloc(&e->d_weights, host.size()) != cudaSuccess) return SF_ENOMEM;
  if (cudaMemcpy(e->d_weights, host.data(), host.size(), cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(e->d_weights);
    return SF_ECUDA;
  }
  for (auto& f : fix) *f.first = static_cast<uint8_t*>(e->d_weights) + f.second;
  // front-end tables and kernel attributes (per device)
  MelTables tab;
  build_mel_tables(&tab);
  if (cudaMalloc(&e->d_mel_tab, sizeof(MelTables)) != cudaSuccess ||
      cudaMemcpy(e->d_mel_tab, &tab, sizeof(tab), cudaMemcpyHostToDevice) != cudaSuccess ||
      frontend_init_attributes() != cudaSuccess || gemm_tc_init_attributes() != cudaSuccess ||
      attention_mha_tc_init_attributes() != cudaSuccess) {
    sf_nem_destroy(e.get());
    e.release();
    return SF_ECUDA;
  }
  // workspace for max_batch clips of max_samples
  const int B = cfg->max_batch;
  const int64_t T_cols = 1 + cfg->max_samples / 160;
  const int64_t Lmax = cfg->max_samples / 160;
  e->M_max = (int64_t)B * ((Lmax + NM_STACK - 1) / NM_STACK);
  const int64_t Mx = e->M_max;
  const size_t sz[] = {(size_t)B * NM_MELS * T_cols * 4, mel_part_floats(B, cfg->max_samples) * 4,
                       (size_t)Mx * NM_D * 4,  (size_t)Mx * 64 * 4,
                       (size_t)Mx * NM_IN * 2, (size_t)Mx * NM_D * 2, (size_t)Mx * NM_FF * 2, (size_t)Mx * NM_D * 2,
                       (size_t)B * 8, sizeof(SeqTable), 256};
  size_t total = 0, offs[11];
  for (int i = 0; i < 11; ++i) {
    offs[i] = total;
    total += (sz[i] + 255) & ~size_t(255);
  }
  if (cudaMalloc(&e->d_ws, total) != cudaSuccess || cudaMallocHost(&e->h_seq, sizeof(SeqTable)) != cudaSuccess) {
    sf_nem_destroy(e.get());
    e.release();
    return SF_ENOMEM;
  }
  uint8_t* w = static_cast<uint8_t*>(e->d_ws);
  e->mel = reinterpret_cast<float*>(w + offs[0]);
  e->part = reinterpret_cast<float*>(w + offs[1]);
  e->x = reinterpret_cast<float*>(w + offs[2]);
  e->logits = reinterpret_cast<float*>(w + offs[3]);
  e->stk = reinterpret_cast<bf16*>(w + offs[4]);
  e->h = reinterpret_cast<bf16*>(w + offs[5]);
  e->big = reinterpret_cast<bf16*>(w + offs[6]);
  e->ctx = reinterpret_cast<bf16*>(w + offs[7]);
  e->d_len = reinterpret_cast<int64_t*>(w + offs[8]);
  e->d_seq = reinterpret_cast<SeqTable*>(w + offs[9]);
  e->d_err = reinterpret_cast<int*>(w + offs[10]);
  if (cudaMemset(e->d_err, 0, 4) != cudaSuccess) {
    sf_nem_destroy(e.get());
    e.release();
    return SF_ECUDA;
  }
  *out = e.release();
  return SF_OK;
}

sf_status sf_nem_destroy(sf_nem_engine* e) {
  if (!e) return SF_EINVAL;
  cudaDeviceSynchronize();
  if (e->d_weights) cudaFree(e->d_weights);
  if (e->d_mel_tab) cudaFree(e->d_mel_tab);
  if (e->d_ws) cudaFree(e->d_ws);
  if (e->h_seq) cudaFreeHost(e->h_seq);
  delete e;
  return SF_OK;
}

const char* sf_nem_last_error(const sf_nem_engine* e) { return e ? e->err.c_str() : "null engine"; }

sf_status sf_nem_forward_offline(sf_nem_engine* e, const float* d_audio, const int64_t* h_len, int B, int64_t n_max,
                                 float* d_probs, int64_t* h_out_len, void* cuda_stream) {
  if (!e) return SF_EINVAL;
  if (!d_audio || !h_len || !d_probs) return nem_fail(e, SF_EINVAL, "null pointer argument");
  if (B < 1 || B > e->cfg.max_batch || n_max < 1600 || n_max > e->cfg.max_samples)
    return nem_fail(e, SF_ESHAPE, "batch or sample count out of range");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != e->device) return nem_fail(e, SF_EDEVICE, "wrong device");
  std::vector<int> tp(B);
  int64_t L_max = n_max / 160;
  int M = 0, max_len = 0, tiles2 = 0;
  SeqTable& sq = *e->h_seq;
  sq.n_seq = B;
  for (int b = 0; b < B; ++b) {
    if (h_len[b] < 1600 || h_len[b] > n_max) return nem_fail(e, SF_EINVAL, "clip length out of range");
    const int64_t L = h_len[b] / 160;
    tp[b] = (int)((L + NM_STACK - 1) / NM_STACK);
    sq.off[b] = M;
    sq.tile_off[b] = 0;
    sq.tile2_off[b] = tiles2;
    M += tp[b];
    tiles2 += (tp[b] + 127) / 128;
    max_len = std::max(max_len, tp[b]);
  }
  sq.off[B] = M;
  sq.tile2_off[B] = tiles2;
  sq.total = M;
  g_launch_pdl = 1;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t ce = cudaSuccess;
#define NCK(x)                    \
  do {                            \
    if ((ce = (x)) != cudaSuccess) \
      goto done;                  \
  } while (0)
  {
    NCK(cudaMemcpyAsync(e->d_len, h_len, (size_t)B * 8, cudaMemcpyHostToDevice, st));
    NCK(cudaMemcpyAsync(e->d_seq, e->h_seq, sizeof(SeqTable), cudaMemcpyHostToDevice, st));
    NCK(launch_mel(d_audio, B, n_max, MelArgs{e->d_len}, e->d_mel_tab, e->mel, e->part, st));
    NCK(launch_k(nem_stack_kernel, dim3(M), dim3(256), 0, st, (const float*)e->mel, (int64_t)(1 + n_max / 160),
                 (const int64_t*)e->d_len, (const SeqTable*)e->d_seq, e->stk));
    NCK(nem_gemm(e, e->stk, NM_IN, e->stack_w, M, NM_D, NM_IN, EPI_F32, e->stack_b, e->x, NM_D, st));
    NCK(launch_layernorm<bf16>(e->x, e->layers[0].ln1_g, e->layers[0].ln1_b, M, NM_D, false, e->h, st));
    const int nl = e->cfg.n_layers;
    for (int l = 0; l < nl; ++l) {
      const NemLayer& w = e->layers[l];
      NCK(nem_gemm(e, e->h, NM_D, w.wqkv, M, 3 * NM_D, NM_D, EPI_BIAS, w.bqkv, e->big, 3 * NM_D, st));
      NCK(launch_k(nem_rope_kernel, dim3((M + 7) / 8), dim3(256), 0, st, e->big, (const SeqTable*)e->d_seq, M));
      NCK(launch_mha_tc_hd64(e->big, e->ctx, e->d_seq, tiles2, M, max_len, NM_D, e->d_err, st));
      NCK(nem_resid_ln(e, e->ctx, NM_D, w.wo, M, NM_D, w.bo, e->x, w.ln2_g, w.ln2_b, e->h, st));
      NCK(nem_gemm(e, e->h, NM_D, w.w1, M, NM_FF, NM_D, EPI_BIAS_SWISH, w.b1, e->big, NM_FF, st));
      const float* g = l + 1 < nl ? e->layers[l + 1].ln1_g : e->fln_g;
      const float* bb = l + 1 < nl ? e->layers[l + 1].ln1_b : e->fln_b;
      NCK(nem_resid_ln(e, e->big, NM_FF, w.w2, M, NM_FF, w.b2, e->x, g, bb, e->h, st));
    }
    NCK(nem_gemm(e, e->h, NM_D, e->head_w, M, NM_UP * NM_SPK, NM_D, EPI_F32, e->head_b, e->logits, NM_UP * NM_SPK,
                 st));
    NCK(cudaMemsetAsync(d_probs, 0, (size_t)B * L_max * NM_SPK * 4, st));
    const int64_t n_el = (int64_t)M * NM_UP * NM_SPK;
    NCK(launch_k(nem_head_out_kernel, dim3((unsigned)((n_el + 255) / 256)), dim3(256), 0, st, (const float*)e->logits,
                 (const int64_t*)e->d_len, (const SeqTable*)e->d_seq, M, L_max, d_probs));
    // device error word: a bounded wait that gave up inside a kernel
    int herr = 0;
    NCK(cudaMemcpyAsync(&herr, e->d_err, 4, cudaMemcpyDeviceToHost, st));
    NCK(cudaStreamSynchronize(st));
    if (herr) {
      cudaMemset(e->d_err, 0, 4);
      return nem_fail(e, (herr & ERR_TIMEOUT) ? SF_ETIMEOUT : SF_ECUDA, "a bounded device wait gave up");
    }
  }
#undef NCK
done:
  if (ce != cudaSuccess) return nem_fail(e, SF_ECUDA, std::string("CUDA: ") + cudaGetErrorString(ce));
  if (h_out_len)
    for (int b = 0; b < B; ++b) h_out_len[b] = h_len[b] / 160;
  return SF_OK;
}

}  // extern "C"
