// sf_mel_noalloc: the log-mel front-end without any allocation.
//
// Who needs it: callers that may not allocate device memory at the point
// where they compute features -- a host process whose memory is budgeted up
// front by a pool or arena allocator it does not control, a plugin that runs
// inside another framework's CUDA context, or a real-time audio thread that
// must not block on cudaMalloc/cudaFree (both can synchronise the device).
// sf_mel needs an engine, whose workspace grows with cudaMalloc; this entry
// point needs no engine and allocates nothing.
//
// Its scratch -- the per-tile statistics the normalisation pass merges, and
// the clip lengths the kernels read -- lives in one file-scope
// `static __device__` array of fixed size (below).  Every GPU that loads
// this library holds that array until the process exits.  In host code the
// array's name is only a host-side stand-in, so its device address is taken
// with cudaGetSymbolAddress, once per device, with that device current, the
// first time the entry point is called on that device; that first call also
// uploads the (host-computed) FFT/window/filterbank tables into a second
// static array with a blocking copy.
//
// All calls share the one array and it keeps the last call's contents: two
// calls whose GPU work overlaps (different streams, or different threads
// without ordering) race on it and corrupt each other's results.  Nothing in
// it needs clearing: each call overwrites the lengths it uses, and the
// statistics kernel writes every (clip, tile, bin) entry it later reads.
#include <mutex>

#include "../../include/sf.h"
#include "common.cuh"
#include "frontend.h"

namespace {

constexpr int NOALLOC_MAX_CLIPS = 64;
// Sum over clips of ceil((1 + n_max / 160) / 32) frame tiles, e.g. 10 clips
// of 120 s (376 tiles each) or one clip of 21.8 minutes.
constexpr int NOALLOC_MAX_TILES = 4096;
constexpr int LEN_FLOATS = NOALLOC_MAX_CLIPS * 2;                 // int64 lengths stored first
// per-tile partial statistics (4 floats per tile and bin), then the per-clip
// (mean, 1 / (std + eps)) of each bin that front-end path 1 writes after them
constexpr size_t PART_FLOATS = (size_t)NOALLOC_MAX_TILES * 128 * 4 + (size_t)NOALLOC_MAX_CLIPS * 128 * 2;
constexpr size_t SCRATCH_FLOATS = LEN_FLOATS + PART_FLOATS;         // 8.06 MiB

static __device__ __align__(256) float g_mel_scratch[SCRATCH_FLOATS];
static __device__ __align__(256) sf::MelTables g_mel_noalloc_tables;

struct DeviceSlot {
  bool ready = false;
  float* scratch = nullptr;
  sf::MelTables* tables = nullptr;
};
constexpr int MAX_DEVICES = 64;
DeviceSlot g_slots[MAX_DEVICES];
std::mutex g_mu;

sf_status setup_device(int dev, DeviceSlot** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceSlot& s = g_slots[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mel_scratch) != cudaSuccess || !p) return SF_ECUDA;
    s.scratch = static_cast<float*>(p);
    p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mel_noalloc_tables) != cudaSuccess || !p) return SF_ECUDA;
    s.tables = static_cast<sf::MelTables*>(p);
    sf::MelTables host;
    sf::build_mel_tables(&host);
    if (cudaMemcpyToSymbol(g_mel_noalloc_tables, &host, sizeof(host)) != cudaSuccess) return SF_ECUDA;
    // per-device: the frame kernels need more than 48 KB of dynamic shared memory
    if (sf::frontend_init_attributes() != cudaSuccess) return SF_ECUDA;
    s.ready = true;
  }
  *out = &s;
  return SF_OK;
}

}  // namespace

extern "C" SF_API sf_status sf_mel_noalloc(const float* d_audio, const int64_t* h_len, int B, int64_t n_max,
                                           float* d_mel, int64_t* h_mel_len, void* cuda_stream) {
  if (!d_audio || !h_len || !d_mel) return SF_EINVAL;
  if (B < 1 || B > NOALLOC_MAX_CLIPS || n_max < 1600) return SF_ESHAPE;
  const int64_t tiles_per_clip = (1 + n_max / 160 + 31) / 32;
  if (tiles_per_clip * B > NOALLOC_MAX_TILES) return SF_ESHAPE;
  if (sf::mel_part_floats(B, n_max) > PART_FLOATS) return SF_ESHAPE;
  for (int b = 0; b < B; ++b)
    if (h_len[b] < 1600 || h_len[b] > n_max) return SF_EINVAL;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return SF_EDEVICE;
  DeviceSlot* slot = nullptr;
  sf_status s = setup_device(dev, &slot);
  if (s != SF_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int64_t* d_len = reinterpret_cast<int64_t*>(slot->scratch);
  float* d_part = slot->scratch + LEN_FLOATS;
  // the lengths go into the scratch with a stream-ordered copy (no allocation)
  if (cudaMemcpyAsync(d_len, h_len, (size_t)B * sizeof(int64_t), cudaMemcpyHostToDevice, st) != cudaSuccess)
    return SF_ECUDA;
  sf::MelArgs args{d_len};
  // the engine's default front-end path, so the result equals sf_mel's to the bit
  if (sf::launch_mel(d_audio, B, n_max, args, slot->tables, d_mel, d_part, st, sf::MEL_DEFAULT_PATH) != cudaSuccess)
    return SF_ECUDA;
  if (h_mel_len)
    for (int b = 0; b < B; ++b) h_mel_len[b] = h_len[b] / 160;
  return SF_OK;
}
