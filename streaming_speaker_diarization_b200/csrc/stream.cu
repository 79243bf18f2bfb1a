// Streaming state machine on the device ("Streaming Sortformer Diarizer",
// Streaming Architecture; NeMo Speaker Diarization API,
// forward_streaming_step and its SortformerStreamingState fields).
//
// assemble:     packed encoder input [cache | FIFO | new frames] per stream.
// state_update: one CTA per stream.  FIFO predictions are refreshed from the
//   window and the chunk is pushed; when the FIFO overflows, its oldest
//   frames pop: silent ones (all probabilities < 0.5) update the running
//   silence mean, and the popped frames join the cache.  If the cache would
//   exceed its length it is compressed: masked log-odds scores, per-speaker
//   top-k by (score desc, index asc) computed as exact ranks, kept frames in
//   candidate order, then silence placeholders in speaker order.
// select_topk:  the selection step alone (teacher-forced checks).
#include <math.h>

#include "stream.h"

namespace sf {

template <typename T>
__global__ void __launch_bounds__(128) assemble_kernel(float* __restrict__ x, const SeqTable* __restrict__ seq,
                                                       const StepDesc* __restrict__ sd, StateBufs sb,
                                                       const T* __restrict__ emb, int emb_stride) {
  SF_PDL_ENTRY();
  const int r = blockIdx.x;
  const int D = sb.D;
  const int i = seq_of_row(seq, r);
  const int loc = r - seq->off[i];
  const int sid = sd->stream[i], n_c = sd->n_c[i], n_f = sd->n_f[i];
  const T* src;
  if (loc < n_c)
    src = reinterpret_cast<const T*>(sb.cache_emb[sd->cur_c[i]]) + ((int64_t)sid * sb.cap_c + loc) * D;
  else if (loc < n_c + n_f)
    src = reinterpret_cast<const T*>(sb.fifo_emb[sd->cur_f[i]]) + ((int64_t)sid * sb.cap_f + loc - n_c) * D;
  else
    src = emb + ((int64_t)i * emb_stride + sd->lc[i] + loc - n_c - n_f) * D;
  float* dst = x + (int64_t)r * D;
  for (int c = threadIdx.x; c < D; c += blockDim.x) dst[c] = to_f<T>(src[c]);
}

template <typename T>
cudaError_t launch_assemble(float* x, const SeqTable* seq, const StepDesc* sd, const StateBufs& sb, const T* emb,
                            int emb_stride, int M, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(assemble_kernel<T>, dim3(M), dim3(128), 0, st, x, seq, sd, sb, emb, emb_stride));
  return cudaGetLastError();
}

// Masked log-odds score of candidate preds p[0..3] (fp32).
__device__ __forceinline__ void masked_scores(const float* p, float* out) {
  int top = 0;
#pragma unroll
  for (int s = 1; s < 4; ++s)
    if (p[s] > p[top]) top = s;
  float l1m[4], lo[4], tot = 0.f;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const float pc = fminf(fmaxf(p[s], 1e-6f), 1.f - 1e-6f);
    l1m[s] = logf(1.f - pc);
    lo[s] = logf(pc / (1.f - pc));
    tot += l1m[s];
  }
#pragma unroll
  for (int s = 0; s < 4; ++s) out[s] = (s == top && p[top] > 0.5f) ? lo[s] + (tot - l1m[s]) : -INFINITY;
}

// Exact per-speaker top-k over sc[n][4] in shared memory.  kept[t] = bit
// mask of the speakers that keep frame t; then slot sources src[0 .. 4k):
// kept frames in ascending index (a frame kept by two speakers appears
// twice), then placeholders -1 - s in speaker order.
__device__ void select_core(const float* sc, int n, int k, int* kept, int* src, int* cnt) {
  for (int t = threadIdx.x; t < n; t += blockDim.x) kept[t] = 0;
  if (threadIdx.x < 4) cnt[threadIdx.x] = 0;
  __syncthreads();
  for (int idx = threadIdx.x; idx < n * 4; idx += blockDim.x) {
    const int t = idx >> 2, s = idx & 3;
    const float v = sc[idx];
    if (!(v > -INFINITY)) continue;
    int rank = 0;
    for (int t2 = 0; t2 < n && rank < k; ++t2) {
      const float v2 = sc[t2 * 4 + s];
      rank += (v2 > v) || (v2 == v && t2 < t);
    }
    if (rank < k) atomicOr(&kept[t], 1 << s);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int p = 0;
    int per[4] = {0, 0, 0, 0};
    for (int t = 0; t < n; ++t)
      for (int s = 0; s < 4; ++s)
        if (kept[t] & (1 << s)) {
          src[p++] = t;
          per[s]++;
        }
    for (int s = 0; s < 4; ++s)
      for (int j = per[s]; j < k; ++j) src[p++] = -1 - s;
    for (int s = 0; s < 4; ++s) cnt[s] = per[s];
  }
  __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(256) state_update_kernel(const float* __restrict__ probs,
                                                           const SeqTable* __restrict__ seq,
                                                           const StepDesc* __restrict__ sd, StateBufs sb,
                                                           const T* __restrict__ emb, int emb_stride,
                                                           float* scores_out, int* src_out,
                                                           const float* scores_in, int score_stride) {
  SF_PDL_ENTRY();
  __shared__ float sc[CAND_MAX * 4];
  __shared__ int kept[CAND_MAX];
  __shared__ int src[CAND_MAX];
  __shared__ int cnt[4];
  __shared__ int n_sil;
  const int i = blockIdx.x;
  const int D = sb.D;
  const int sid = sd->stream[i], n_c = sd->n_c[i], n_f = sd->n_f[i], cl = sd->cl[i], npop = sd->npop[i];
  const int cc = sd->cur_c[i], cf = sd->cur_f[i];
  if (sd->n_new[i] <= 0) return;   // finished stream: nothing to update
  T* cache = reinterpret_cast<T*>(sb.cache_emb[cc]) + (int64_t)sid * sb.cap_c * D;
  float* cpred = sb.cache_preds[cc] + (int64_t)sid * sb.cap_c * 4;
  T* fifo = reinterpret_cast<T*>(sb.fifo_emb[cf]) + (int64_t)sid * sb.cap_f * D;
  float* fpred = sb.fifo_preds[cf] + (int64_t)sid * sb.cap_f * 4;
  const T* newe = emb + ((int64_t)i * emb_stride + sd->lc[i]) * D;
  const float* wp = probs + (int64_t)(seq->off[i] + n_c) * 4;   // FIFO rows then chunk rows
  const int nF = n_f + cl;
  auto femb = [&](int t) -> const T* { return t < n_f ? fifo + (int64_t)t * D : newe + (int64_t)(t - n_f) * D; };

  if (npop == 0) {
    for (int e = threadIdx.x; e < nF * 4; e += blockDim.x) fpred[e] = wp[e];
    for (int e = threadIdx.x; e < cl * D; e += blockDim.x) fifo[(int64_t)n_f * D + e] = newe[e];
    return;
  }
  // pop: the remaining FIFO frames go to the other FIFO buffer
  T* fifo_new = reinterpret_cast<T*>(sb.fifo_emb[cf ^ 1]) + (int64_t)sid * sb.cap_f * D;
  float* fpred_new = sb.fifo_preds[cf ^ 1] + (int64_t)sid * sb.cap_f * 4;
  const int nrem = nF - npop;
  for (int e = threadIdx.x; e < nrem * 4; e += blockDim.x) fpred_new[e] = wp[npop * 4 + e];
  for (int t = 0; t < nrem; ++t) {
    const T* s = femb(npop + t);
    for (int c = threadIdx.x; c < D; c += blockDim.x) fifo_new[(int64_t)t * D + c] = s[c];
  }
  // silence statistics of the popped frames
  for (int t = threadIdx.x; t < npop; t += blockDim.x)
    kept[t] = (wp[t * 4] < 0.5f && wp[t * 4 + 1] < 0.5f && wp[t * 4 + 2] < 0.5f && wp[t * 4 + 3] < 0.5f) ? 1 : 0;
  if (threadIdx.x == 0) n_sil = 0;
  __syncthreads();
  if (threadIdx.x == 0) {
    int m = 0;
    for (int t = 0; t < npop; ++t) m += kept[t];
    n_sil = m;
  }
  __syncthreads();
  float* sil = sb.sil_mean + (int64_t)sid * D;
  const int m = n_sil;
  if (m > 0) {
    const int c0 = sb.sil_count[sid];
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
      float s = 0.f;
      for (int t = 0; t < npop; ++t)
        if (kept[t]) s += to_f<T>(femb(t)[c]);
      sil[c] = (sil[c] * (float)c0 + s) / (float)(c0 + m);
    }
    __syncthreads();
    if (threadIdx.x == 0) sb.sil_count[sid] = c0 + m;
  }
  const int nC = n_c + npop;
  if (nC <= sb.cache_len) {
    for (int e = threadIdx.x; e < npop * 4; e += blockDim.x) cpred[n_c * 4 + e] = wp[e];
    for (int t = 0; t < npop; ++t) {
      const T* s = femb(t);
      for (int c = threadIdx.x; c < D; c += blockDim.x) cache[(int64_t)(n_c + t) * D + c] = s[c];
    }
    return;
  }
  // compression
  __syncthreads();
  for (int t = threadIdx.x; t < nC; t += blockDim.x) {
    const float* p = t < n_c ? cpred + t * 4 : wp + (t - n_c) * 4;
    float o[4];
    if (scores_in) {
#pragma unroll
      for (int s = 0; s < 4; ++s) o[s] = scores_in[((int64_t)i * score_stride + t) * 4 + s];
    } else {
      masked_scores(p, o);
    }
#pragma unroll
    for (int s = 0; s < 4; ++s) sc[t * 4 + s] = o[s];
    if (scores_out) {
#pragma unroll
      for (int s = 0; s < 4; ++s) scores_out[((int64_t)i * score_stride + t) * 4 + s] = o[s];
    }
  }
  __syncthreads();
  const int k = sb.cache_len / 4;
  select_core(sc, nC, k, kept, src, cnt);
  T* cache_new = reinterpret_cast<T*>(sb.cache_emb[cc ^ 1]) + (int64_t)sid * sb.cap_c * D;
  float* cpred_new = sb.cache_preds[cc ^ 1] + (int64_t)sid * sb.cap_c * 4;
  const int n_slots = 4 * k;
  for (int p = 0; p < n_slots; ++p) {
    const int t = src[p];
    if (t >= 0) {
      const T* s = t < n_c ? cache + (int64_t)t * D : femb(t - n_c);
      for (int c = threadIdx.x; c < D; c += blockDim.x) cache_new[(int64_t)p * D + c] = s[c];
    } else {
      for (int c = threadIdx.x; c < D; c += blockDim.x) cache_new[(int64_t)p * D + c] = from_f<T>(sil[c]);
    }
  }
  for (int e = threadIdx.x; e < n_slots * 4; e += blockDim.x) {
    const int p = e >> 2, s = e & 3, t = src[p];
    cpred_new[e] = t < 0 ? 0.f : (t < n_c ? cpred[t * 4 + s] : wp[(t - n_c) * 4 + s]);
  }
  if (src_out)
    for (int p = threadIdx.x; p < n_slots; p += blockDim.x) src_out[(int64_t)i * sb.cache_len + p] = src[p];
}

template <typename T>
cudaError_t launch_state_update(const float* probs, const SeqTable* seq, const StepDesc* sd, StateBufs sb,
                                const T* emb, int emb_stride, int n_seq, float* scores_out, int* src_out,
                                const float* scores_in, int score_stride, cudaStream_t st) {
  if (n_seq <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(state_update_kernel<T>, dim3(n_seq), dim3(256), 0, st, probs, seq, sd, sb, emb, emb_stride, scores_out, src_out, scores_in,
                                                score_stride));
  return cudaGetLastError();
}

__global__ void __launch_bounds__(256) select_topk_kernel(const float* __restrict__ scores, const int* __restrict__ n,
                                                          int stride, int k, int* __restrict__ src_out) {
  SF_PDL_ENTRY();
  __shared__ float sc[CAND_MAX * 4];
  __shared__ int kept[CAND_MAX];
  __shared__ int src[CAND_MAX];
  __shared__ int cnt[4];
  const int i = blockIdx.x;
  const int nn = n[i];
  for (int e = threadIdx.x; e < nn * 4; e += blockDim.x) sc[e] = scores[(int64_t)i * stride * 4 + e];
  __syncthreads();
  select_core(sc, nn, k, kept, src, cnt);
  for (int p = threadIdx.x; p < 4 * k; p += blockDim.x) src_out[(int64_t)i * 4 * k + p] = src[p];
}

cudaError_t launch_select_topk(const float* scores, const int* n, int n_sets, int stride, int k, int* src,
                               cudaStream_t st) {
  if (n_sets <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(select_topk_kernel, dim3(n_sets), dim3(256), 0, st, scores, n, stride, k, src));
  return cudaGetLastError();
}

template cudaError_t launch_assemble<float>(float*, const SeqTable*, const StepDesc*, const StateBufs&, const float*, int, int, cudaStream_t);
template cudaError_t launch_assemble<bf16>(float*, const SeqTable*, const StepDesc*, const StateBufs&, const bf16*, int, int, cudaStream_t);
template cudaError_t launch_state_update<float>(const float*, const SeqTable*, const StepDesc*, StateBufs, const float*, int, int, float*, int*, const float*, int, cudaStream_t);
template cudaError_t launch_state_update<bf16>(const float*, const SeqTable*, const StepDesc*, StateBufs, const bf16*, int, int, float*, int*, const float*, int, cudaStream_t);

}  // namespace sf
