// Streaming-state kernels: descriptors and launchers.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace sf {

constexpr int CAND_MAX = 1024;   // compression candidates per stream (cache + popped)

// Per-sequence description of one streaming step (device memory).  For
// offline calls n_c = n_f = lc = 0 and n_new = the clip's frames.
struct StepDesc {
  int stream[MAX_SEQ];   // state slot of sequence i
  int n_c[MAX_SEQ];      // cache rows before the step
  int n_f[MAX_SEQ];      // FIFO rows before the step
  int lc[MAX_SEQ];       // left-context frames to drop from the window's embeddings
  int n_new[MAX_SEQ];    // new frames (chunk + look-ahead)
  int cl[MAX_SEQ];       // chunk frames emitted and pushed to the FIFO
  int npop[MAX_SEQ];     // frames popped from the FIFO (0 = none)
  int first_out[MAX_SEQ];// n_c + n_f (first emitted row of the window)
  int cur_c[MAX_SEQ];    // which cache buffer (0/1) holds the state
  int cur_f[MAX_SEQ];    // which FIFO buffer (0/1) holds the state
};

// Device-resident state of a stream batch (double-buffered cache and FIFO).
struct StateBufs {
  void* cache_emb[2];    // act [n_streams x cap_c x D]
  float* cache_preds[2]; // [n_streams x cap_c x 4]
  void* fifo_emb[2];     // act [n_streams x cap_f x D]
  float* fifo_preds[2];  // [n_streams x cap_f x 4]
  float* sil_mean;       // [n_streams x D]
  int* sil_count;        // [n_streams]
  int cap_c, cap_f, D;
  int cache_len;         // preset spkcache_len
};

// x[row] = f32([cache | FIFO | new frames][row]) for every packed row.
template <typename T>
cudaError_t launch_assemble(float* x, const SeqTable* seq, const StepDesc* sd, const StateBufs& sb, const T* emb,
                            int emb_stride, int M, cudaStream_t st);

// State update after the encoder: one CTA per sequence.  probs [M x 4]
// packed window predictions; emb act [n x emb_stride x D] window embeddings.
// scores_out / src_out optional debug outputs; scores_in optional override.
template <typename T>
cudaError_t launch_state_update(const float* probs, const SeqTable* seq, const StepDesc* sd, StateBufs sb,
                                const T* emb, int emb_stride, int n_seq, float* scores_out, int* src_out,
                                const float* scores_in, int score_stride, cudaStream_t st);

// Standalone per-speaker top-k: one CTA per set.
cudaError_t launch_select_topk(const float* scores, const int* n, int n_sets, int stride, int k, int* src,
                               cudaStream_t st);

}  // namespace sf
