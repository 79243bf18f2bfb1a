// Post-processing of frame probabilities into speaker segments ("Streaming
// Sortformer Diarizer" model card, Output: VAD-style thresholding and
// smoothing into [start_seconds, end_seconds, speaker_index]).
//
// One warp per (clip, speaker).  Hysteresis binarisation, 32 frames at a
// time: a frame is decisive when p > onset (on) or p <= offset (off); every
// other frame keeps the state of the frame before it, so a lane's state is
// the on-bit of the nearest decisive lane at or before it (ballots + count-
// leading-zeros), or the carry from the previous 32 frames.  Run starts and
// ends are the transitions of that state mask, taken in frame order by the
// whole warp; each run is padded, merged with the previous segment when it
// starts at or before its end or within min_duration_off of it, and a
// finished segment is kept if it lasts at least min_duration_on.  Times are
// float64 with every product and sum rounded separately (no fused
// multiply-add), so they equal a plain evaluation of the same expressions.
#include "common.cuh"
#include "layers.h"

namespace sf {

__global__ void __launch_bounds__(128) segments_kernel(const float* __restrict__ probs, int stride_t,
                                                       const int* __restrict__ n_frames, SegArgs a,
                                                       double* __restrict__ segs, int* __restrict__ counts) {
  const int clip = blockIdx.x, spk = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = n_frames[clip];
  const float* p = probs + (int64_t)clip * stride_t * 4 + spk;
  double* out = segs + ((int64_t)clip * 4 + spk) * a.max_seg * 2;
  const double dur = __dmul_rn((double)T, 0.08);
  int count = 0;
  bool have = false;
  double ps = 0.0, pe = 0.0;
  auto flush = [&]() {
    if (__dsub_rn(pe, ps) >= a.min_on) {
      if (count < a.max_seg && lane == 0) {
        out[2 * count] = ps;
        out[2 * count + 1] = pe;
      }
      ++count;
    }
  };
  auto emit_run = [&](int r0, int r1) {   // frames r0 .. r1 active
    const double s = fmax(__dsub_rn(__dmul_rn((double)r0, 0.08), a.pad_on), 0.0);
    const double e = fmin(__dadd_rn(__dmul_rn((double)(r1 + 1), 0.08), a.pad_off), dur);
    if (have && (s <= pe || __dsub_rn(s, pe) < a.min_off)) {
      pe = fmax(pe, e);
    } else {
      if (have) flush();
      ps = s;
      pe = e;
      have = true;
    }
  };
  uint32_t state = 0;   // activity of the frame before this block of 32
  int run_start = 0;
  const uint32_t upto = lane == 31 ? 0xffffffffu : ((2u << lane) - 1u);
  for (int base = 0; base < T; base += 32) {
    const int t = base + lane;
    const bool valid = t < T;
    const float v = valid ? p[(int64_t)t * 4] : 0.f;
    const uint32_t on_b = __ballot_sync(0xffffffffu, valid && v > a.onset);
    // frames past the clip end are decisive and inactive
    const uint32_t dec_b = __ballot_sync(0xffffffffu, !valid || v > a.onset || v <= a.offset);
    const uint32_t d = dec_b & upto;
    const uint32_t st = d ? (on_b >> (31 - __clz(d))) & 1u : state;
    const uint32_t s_b = __ballot_sync(0xffffffffu, st != 0);
    const uint32_t prev_b = (s_b << 1) | state;
    const uint32_t starts = s_b & ~prev_b, ends = ~s_b & prev_b;
    uint32_t ev = starts | ends;
    while (ev) {   // warp-uniform: every lane walks the same transitions
      const int l = __ffs(ev) - 1;
      ev &= ev - 1;
      if ((starts >> l) & 1u) run_start = base + l;
      else emit_run(run_start, base + l - 1);
    }
    state = s_b >> 31;
  }
  if (state) emit_run(run_start, T - 1);   // T a multiple of 32, active to the end
  if (have) flush();
  if (lane == 0) counts[clip * 4 + spk] = count;
}

cudaError_t launch_segments(const float* probs, int stride_t, const int* d_n_frames, int n, const SegArgs& a,
                            double* segs, int* counts, cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  CK_LAUNCH(launch_k(segments_kernel, dim3(n), dim3(128), 0, st, probs, stride_t, d_n_frames, a, segs, counts));
  return cudaGetLastError();
}

}  // namespace sf
