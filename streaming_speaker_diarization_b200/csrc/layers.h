// Launchers of the engine's kernels (host-callable, stream-ordered).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace sf {

// ------------------------------------------------------------------ GEMM
enum EpiKind : int {
  EPI_BIAS = 0,        // out(act) = acc + b
  EPI_BIAS_RELU = 1,   // out(act) = relu(acc + b)
  EPI_BIAS_SWISH = 2,  // out(act) = swish(acc + b)
  EPI_BIAS_GLU = 3,    // columns (2c, 2c+1) = (a_c, g_c): out(act)[c] = a_c * sigmoid(g_c)
  EPI_RESID = 4,       // out(f32) += alpha * (acc + b)
  EPI_F32 = 5,         // out(f32) = acc + b
  EPI_F32_AND_T = 6,   // out(f32) = acc + b and out2(act) = acc + b
  EPI_RESID_LN = 7,    // x_new = out(f32) + alpha * (acc + b), then LayerNorm over each full row:
                       //   ln_xnorm 0: out <- x_new,     ln_h <- act(LN(x_new))
                       //   ln_xnorm 1: out <- LN(x_new), ln_h <- act(LN2(LN(x_new))) with ln_g2,
                       //               else act(LN(x_new))
                       // (bf16 tcgen05 path only; the N tiles of a row block form a CTA cluster)
};

struct Epi {
  int kind;
  const float* bias;   // [N] or null
  void* out;
  int ldo;             // elements
  float alpha;
  void* out2;
  int ldo2;
  int rpg;             // row remap: 0 = identity, else row r -> (r / rpg) * gstride + r % rpg
  int64_t gstride;
  // EPI_RESID_LN: LayerNorm weights (length N), optional second LayerNorm,
  // the act output [M x ldh] and whether out receives the normalised row
  const float* ln_g;
  const float* ln_b;
  const float* ln_g2;
  const float* ln_b2;
  void* ln_h;
  int ldh;
  int ln_xnorm;
};

cudaError_t gemm_f32(const float* A, int lda, const float* W, int M, int N, int K, const Epi& e, cudaStream_t st);
cudaError_t gemm_bf16_mma(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e,
                          cudaStream_t st);
cudaError_t gemm_init_attributes();
// Scratch of the tcgen05 GEMM: error word, split-K partial tiles and the
// per-tile arrival counters (zero between launches; the last CTA of a tile
// resets its counter).  ws/cnt may be null: no split-K then.
struct TcScratch {
  int* err;
  float* ws;
  size_t ws_bytes;
  int* cnt;
  int cnt_len;
};
// tcgen05 / TMEM / TMA path (sm_100a).
cudaError_t gemm_bf16_tc(const bf16* A, int lda, const bf16* W, int M, int N, int K, const Epi& e,
                         const TcScratch& sc, cudaStream_t st);
cudaError_t gemm_tc_init_attributes();
// 2-D bf16 tensor map (row-major [rows x cols], row stride ld elements), box
// box_rows x 64 columns, 128-byte swizzle, zero fill outside the matrix.
cudaError_t make_bf16_map_sw128(CUtensorMap* m, const void* base, int rows, int cols, int ld, int box_rows);
// Multi-wave bf16 GEMMs on the CTA-pair (cta_group::2) kernel: 0 never, 1
// where it is faster (K >= 1024, N >= 256), 2 always; set from the calling
// engine's options at each API entry.
extern int g_gemm_pairs;
// Pair tile width forced for those GEMMs (128, 192 or 256); 0 = planned.
extern int g_gemm_pair_bn;
void gemm_tc_plan(int M, int N, int K, const TcScratch& sc, int* bn, int* splits);
// Whether an EPI_RESID_LN GEMM of this shape runs fused: N a multiple of 64
// with at most 8 tiles of 64 (one cluster per 128-row block) and every
// cluster co-resident (one wave); otherwise use EPI_RESID and a LayerNorm.
bool gemm_ln_fusable(int M, int N, int K);

// --------------------------------------------------------- subsampling
struct PreArgs {        // device arrays, one entry per window
  const int* buf;       // feature buffer row
  const int64_t* start; // first column
  const int64_t* frames;// window length W (mel frames)
};

template <typename T>
cudaError_t launch_conv1(const float* feats, int64_t t_buf, const PreArgs& a, int n_win, const float* w,
                         const float* b, T* out, int T1max, cudaStream_t st);
template <typename T>
cudaError_t launch_dwconv3x3s2(const T* in, int Tin_max, int Fin, T* out, int Tout_max, int Fout, const PreArgs& a,
                               int n_win, int stage, const float* w, const float* b, cudaStream_t st);
// conv1 (w1, b1) and the first depthwise stage (w2, b2) in one pass: out
// [n_win][T2max][32][256], equal to launch_conv1 followed by
// launch_dwconv3x3s2(stage 1) without the stage-1 tensor.
template <typename T>
cudaError_t launch_conv1_dw(const float* feats, int64_t t_buf, const PreArgs& a, int n_win, const float* w1,
                            const float* b1, const float* w2, const float* b2, T* out, int T2max, cudaStream_t st);

// ------------------------------------------------------- norms / elementwise
// x (f32, M x D) -> optional in-place LN(x) (f32) and/or h = act(LN(x)).
// With g2/b2: x <- LN1(x) and h = act(LN2(LN1(x))) in one pass.
template <typename T>
cudaError_t launch_layernorm(float* x, const float* g, const float* b, int M, int D, bool write_x, T* h,
                             cudaStream_t st, const float* g2 = nullptr, const float* b2 = nullptr);
// Conformer depthwise conv (k=9, zero padding at sequence edges) with the
// folded BatchNorm and swish: in/out act (M x D).
template <typename T>
cudaError_t launch_dwconv1d(const T* in, T* out, const float* w, const float* b, int M, int D, int K,
                            const SeqTable* seq, cudaStream_t st);
// Head output layer: probs[r][s] = sigmoid(h[r] . w[s] + b[s]), w f32 (4 x E).
template <typename T>
cudaError_t launch_head_out(const T* h, const float* w, const float* b, float* probs, int M, int E,
                            cudaStream_t st);
// Packed embeddings (act, M x D) -> f32 residual stream.
template <typename T>
cudaError_t launch_to_f32(const T* in, float* out, int64_t n, cudaStream_t st);
// out[s][t][0..3] = t < count_s ? packed[off_s + first_s + t][0..3] : 0 for t < t_max
// (d_first null = 0, d_count null = sequence length).
// d_dst (null = identity) gives the output row block of each sequence.
cudaError_t launch_extract_rows(const float* packed, const SeqTable* seq, const int* d_first, const int* d_count,
                                const int* d_dst, int n_seq, float* out, int t_max, cudaStream_t st);
// fp32 attention: sequences up to attention_f32_max_seq() rows (one score
// row per warp in shared memory); attention_reserve_f32(R) raises the
// kernels' shared-memory limit to cover R rows (never lowers it).
int attention_f32_max_seq();
cudaError_t attention_reserve_f32(int R);

// One CTA waits on an mbarrier nothing arrives on, through the tcgen05
// kernels' bounded wait; when it gives up, ERR_TIMEOUT goes to *err.
cudaError_t launch_selftest_wait(int* err, cudaStream_t st);

// ------------------------------------------------------- post-processing
struct SegArgs {
  float onset, offset;      // activity thresholds (onset >= offset)
  double pad_on, pad_off;   // seconds added before / after each run
  double min_on, min_off;   // shortest kept segment, shortest kept gap (s)
  int max_seg;              // segments stored per (clip, speaker)
};
// probs f32 [n][stride_t][4], d_n_frames i32 [n] -> segs f64
// [n][4][max_seg][2] (start, end seconds), counts i32 [n][4] (found, may
// exceed max_seg; only the first max_seg are stored).
cudaError_t launch_segments(const float* probs, int stride_t, const int* d_n_frames, int n, const SegArgs& a,
                            double* segs, int* counts, cudaStream_t st);

// ------------------------------------------------------------- attention
// Relative-position MHSA (d_model 512, 8 heads of 64) over packed sequences.
//   qkv act [M x 3*512] (q | k | v), ptab act [(2R-1) x 512] projected
//   sinusoid rows for r = -(R-1) .. R-1, u/v f32 [8 x 64]; ctx act [M x 512].
template <typename T>
cudaError_t launch_relpos_attention(const T* qkv, const T* ptab, int R, const float* u, const float* v, T* ctx,
                                    const SeqTable* seq, int n_tiles, int M, cudaStream_t st);
// Plain MHSA (d 192, 8 heads of 24), qkv act [M x 576] -> ctx act [M x 192];
// R bounds the sequence lengths (used by the fp32 kernel's score rows).
template <typename T>
cudaError_t launch_mha(const T* qkv, T* ctx, const SeqTable* seq, int n_tiles, int M, int R, cudaStream_t st);
cudaError_t attention_init_attributes();
// bf16 relative-position MHSA on tcgen05 (one CTA per 128 query rows x head
// x key split; n_tiles2 = 128-row tiles of the sequence table, max_len the
// longest sequence); with fewer (tile, head) units than SMs each unit's keys
// are split over a cluster of 2 or 4 CTAs merged in shared memory; sc.err
// gets ERR_TIMEOUT if a bounded wait gives up.
cudaError_t launch_relpos_attention_tc(const bf16* qkv, const bf16* ptab, int R, const float* u, const float* v,
                                       bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                                       const TcScratch& sc, cudaStream_t st);
cudaError_t attention_tc_init_attributes();
// bf16 Transformer MHSA (d 192, 8 heads of 24) on tcgen05: one CTA per 128
// query rows x head x key split (n_tiles2 = 128-row tiles, max_len the
// longest sequence); with fewer units than two per SM each unit's keys are
// split over a cluster of 2 or 4 CTAs merged in shared memory; err gets
// ERR_TIMEOUT if a bounded wait gives up.
cudaError_t launch_mha_tc(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                          int* err, cudaStream_t st);
// The same kernel with heads of 64 (8 heads, E = 512: the Nemotron-3 variant).
cudaError_t launch_mha_tc_hd64(const bf16* qkv, bf16* ctx, const SeqTable* seq, int n_tiles2, int M, int max_len,
                               int E, int* err, cudaStream_t st);
cudaError_t attention_mha_tc_init_attributes();

// ------------------------------------------------- fused Transformer layer
// One post-LN Transformer layer after its attention (d 192, FFN 768 ReLU):
// x <- LN1(x + ctx Wo^T + bo); x <- LN2(x + relu(x W1^T + b1) W2^T + b2);
// then qkv <- x Wqkv'^T + bqkv' of the next layer (next given) or h <- bf16(x).
// One cluster of four CTAs per 128-row block (tcgen05 products, LayerNorm
// statistics and FFN partial sums exchanged in distributed shared memory).
struct TfLayerW {
  const bf16 *wqkv, *wo, *w1, *w2;   // [576 x 192], [192 x 192], [768 x 192], [192 x 768]
  const float *bqkv, *bo, *ln1_g, *ln1_b, *b1, *b2, *ln2_g, *ln2_b;
};
struct TfLayerArgs {
  float* x;
  const float *bo, *ln1_g, *ln1_b, *b1, *b2, *ln2_g, *ln2_b, *bq;
  bf16* qkv;
  bf16* h;
};
cudaError_t launch_tf_layer(const bf16* ctx, const TfLayerW& w, const TfLayerW* next, float* x, bf16* qkv, bf16* h,
                            int M, int* err, cudaStream_t st);
// Rows the fused layer covers in one wave (co-resident clusters x 128).
int tf_layer_max_rows();
cudaError_t tf_layer_init_attributes();

}  // namespace sf
