// Log-mel front-end launchers and tables.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace sf {

constexpr int MEL_MAX_NK = 16;   // FFT bins per Slaney filter (widest is ~13 at 8 kHz)

// Host-computed (double, then rounded) tables for the mel kernels.
struct MelTables {
  float2 tw256[128];             // exp(-2 pi i k / 256)
  float2 tw512[257];             // exp(-2 pi i k / 512)
  float win[512];                // symmetric 400-point Hann centred in 512
  int mel_k0[128];               // first FFT bin of filter m
  int mel_nk[128];               // number of FFT bins of filter m
  float mel_w[128 * MEL_MAX_NK]; // filter weights (area-normalised)
};

struct MelArgs {
  const int64_t* len;            // device [B] clip lengths in samples
  // window mode (all null for whole clips): clip b is frames f0[b] ..
  // f0[b] + nf[b] - 1 of the audio in buffer row row[b], whose column 0 is
  // sample a0[b]; len[b] samples have arrived (zeros beyond); statistics and
  // normalisation over the window's nf[b] frames; features go to row row[b]
  // of the output
  const int64_t* f0 = nullptr;
  const int64_t* a0 = nullptr;
  const int* nf = nullptr;
  const int* row = nullptr;
};

// path 0: shared-memory radix-2 FFT per warp, one normalisation CTA per
// (clip, bin); path 1: register/shuffle FFT, a statistics pass and a
// normalisation pass spread over all SMs.  Same results up to rounding.
// Path 1 is the default (measured 2.1x faster on one hour of audio).
constexpr int MEL_DEFAULT_PATH = 1;
cudaError_t launch_mel(const float* audio, int B, int64_t n_max, const MelArgs& args, const MelTables* tab,
                       float* mel, float* part, cudaStream_t st, int path = MEL_DEFAULT_PATH);
// Window mode: T_cols window columns per clip, buffer rows of n_buf samples.
cudaError_t launch_mel_windows(const float* audio, int B, int64_t n_buf, const MelArgs& args, const MelTables* tab,
                               float* mel, float* part, int T_cols, cudaStream_t st, int path = MEL_DEFAULT_PATH);
// Floats of `part` a call over B clips of up to n_max samples (or windows
// of up to 1 + n_max / 160 columns) needs.
size_t mel_part_floats(int B, int64_t n_max);
cudaError_t frontend_init_attributes();
void build_mel_tables(MelTables* t);   // host

}  // namespace sf
