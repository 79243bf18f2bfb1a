/*
 * sf.h -- C ABI of the B200 Streaming Sortformer diarization engine (libsf.so).
 *
 * The engine computes the forward pass described on the "Streaming Sortformer
 * Diarizer" page (Pipeline): 16 kHz audio -> 128-bin log-mel (25 ms window,
 * 10 ms stride) -> ConvSubsampling 8x -> 17 FastConformer layers (d=512) ->
 * Linear 512->192 -> 18 Transformer layers (d=192, 8 heads) ->
 * Linear-ReLU-Linear-sigmoid head: per-80 ms activity of 4 speakers.  In
 * streaming mode each step runs the encoder on [speaker cache | FIFO | chunk]
 * (page section "Streaming Architecture"; NeMo Speaker Diarization API,
 * forward_streaming_step).
 *
 * Conventions for every call:
 *  - Pointers prefixed d_ are CUDA device memory, h_ are host memory; all
 *    are owned by the caller, who keeps them valid until the call's GPU work
 *    has finished on the given stream.
 *  - Element types: audio, mel features and probabilities are float32.
 *    Embeddings exchanged through sf_pre_encode / sf_encode / the state view
 *    use the engine's precision: float32 in SF_FP32 mode, bfloat16 (raw
 *    uint16 bit patterns) in SF_BF16 mode ("act" type below).
 *  - All arrays are dense row-major with the shapes given.
 *  - `cuda_stream` is a cudaStream_t (NULL = the legacy default stream).
 *    Work is enqueued asynchronously unless a call says it synchronises.
 *  - Return value: SF_OK, or an error code with a message retrievable by
 *    sf_last_error().  Argument and shape checks happen on the host before
 *    any work is enqueued; on such an error nothing is enqueued and no
 *    output is written.  SF_ECUDA reports a launch or runtime error.
 *    SF_ETIMEOUT reports that a bounded device-side wait gave up (the
 *    engine's kernels never spin without a limit).
 *  - An engine or stream object must not be used from two host threads at
 *    once (creating or destroying a stream uses its engine), and calls on
 *    one engine must be ordered: issue them on one CUDA
 *    stream (or order the streams yourself), because every call reuses the
 *    engine's workspace and descriptor block.  Different engines may be
 *    driven from different host threads (e.g. one engine and one thread
 *    per GPU); the GEMM kernel selection (SF_OPT_GEMM_PATH,
 *    SF_OPT_GEMM_PAIR_BN) is then shared by the process, so give those
 *    engines the same values.
 */
#ifndef SF_H_
#define SF_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SF_API __attribute__((visibility("default")))
#else
#define SF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sf_engine sf_engine;
typedef struct sf_stream sf_stream;

typedef enum {
  SF_OK = 0,
  SF_EINVAL = 1,    /* bad argument (null pointer, out-of-range value)      */
  SF_ESHAPE = 2,    /* sizes beyond what the engine was created for         */
  SF_ENOMEM = 3,    /* device or pinned-host allocation failed               */
  SF_ECUDA = 4,     /* CUDA launch / runtime error                           */
  SF_ESTATE = 5,    /* call not valid in the object's current state          */
  SF_ETIMEOUT = 6,  /* a bounded device wait gave up                         */
  SF_EDEVICE = 7,   /* no usable sm_100 device                               */
  SF_EFORMAT = 8    /* weight blob malformed or missing a tensor             */
} sf_status;

typedef enum { SF_FP32 = 0, SF_BF16 = 1 } sf_precision;

/* Model and capacity description ("Streaming Sortformer Diarizer", Model
 * Parameters table; metadata of the exported program: sample_rate,
 * window_stride, subsampling_factor, fc_d_model, tf_d_model,
 * max_num_of_spks, spkcache_len).  Only n_conformer, n_transformer,
 * precision, max_batch and max_samples may differ from sf_default_config();
 * the other fields are checked. */
typedef struct {
  int sample_rate;     /* 16000 */
  int n_mels;          /* 128 */
  int n_fft;           /* 512 */
  int win_length;      /* 400 samples (25 ms) */
  int hop_length;      /* 160 samples (10 ms) */
  int subsampling;     /* 8 */
  int d_model;         /* 512  (fc_d_model) */
  int tf_d_model;      /* 192 */
  int n_conformer;     /* 17 */
  int n_transformer;   /* 18 */
  int n_heads;         /* 8 */
  int ff_mult;         /* 4 (FFN 512 -> 2048) */
  int tf_ff;           /* 768 */
  int conv_kernel;     /* 9 */
  int n_spk;           /* 4 (max_num_of_spks) */
  int spkcache_len;    /* 188 */
  int precision;       /* sf_precision */
  int max_batch;       /* max clips per offline call and streams per sf_stream (<= 512) */
  int64_t max_samples; /* max samples per clip (default 1,920,000 = 120 s) */
} sf_config;

/* Streaming preset, all lengths in 80 ms encoder frames ("Streaming
 * Configurations" table: Very high 340/40/40/300/188, High 124/1/124/124/188,
 * Low 6/7/188/144/188, Ultra low 3/1/188/144/188).  Input-buffer latency is
 * (chunk_len + right_context) x 80 ms. */
typedef struct {
  int chunk_len;
  int right_context;
  int fifo_len;
  int update_period;
  int spkcache_len;    /* <= config spkcache_len, multiple of n_spk */
} sf_preset;

/* State of one stream (NeMo SortformerStreamingState fields spkcache,
 * spkcache_lengths, spkcache_preds, fifo, fifo_lengths, fifo_preds; plus the
 * engine's silence mean used for cache placeholders and the position of the
 * next chunk).  Device buffers are caller-owned; capacities are
 * spkcache_len rows for the cache and fifo_len + chunk_len rows for the
 * FIFO. */
typedef struct {
  int n_cache;          /* rows in the speaker cache */
  int n_fifo;           /* rows in the FIFO */
  int64_t next_frame;   /* encoder frame index of the next chunk (c0) */
  int finished;         /* 1 after the step that consumed the recording end */
  int sil_count;        /* popped silent frames averaged into sil_mean */
  void* d_cache_emb;    /* act [capacity_cache x d_model] pre-encode embeddings */
  float* d_cache_preds; /* f32 [capacity_cache x n_spk] */
  void* d_fifo_emb;     /* act [capacity_fifo x d_model] */
  float* d_fifo_preds;  /* f32 [capacity_fifo x n_spk] */
  float* d_sil_mean;    /* f32 [d_model] */
} sf_state_view;

/* ---------------------------------------------------------------- engine */

/* Fill `cfg` with the full model (17 + 18 layers), bf16, max_batch 64,
 * max_samples 1,920,000. */
SF_API sf_status sf_default_config(sf_config* cfg);

/* Create an engine on the current CUDA device from a weight blob in host
 * memory (SFW1 container: magic "SFW1", u32 tensor count, u64 payload
 * offset, then per tensor u16 name length, name, u8 ndim, u32 dims, u64
 * payload offset; float32 payloads).  Weights are converted to the engine's
 * precision, BatchNorm is folded into the depthwise conv, the relative
 * position projections are precomputed for every distance up to the longest
 * sequence the configuration allows, and the workspace is allocated.  The
 * blob may be freed after the call.  Synchronises.  max_samples may reach
 * 4 h (230,400,000) in bf16; an fp32 engine keeps one attention score row
 * per warp in shared memory, which bounds its sequences to 14,000 encoder
 * frames (max_samples <= 17,920,159, about 18.7 min).  Errors: SF_EINVAL,
 * SF_ESHAPE (fp32 with a longer max_samples), SF_EFORMAT (missing/mis-shaped
 * tensor), SF_EDEVICE, SF_ENOMEM. */
SF_API sf_status sf_create(const void* h_blob, uint64_t nbytes, const sf_config* cfg, sf_engine** out);
SF_API sf_status sf_create_from_file(const char* path, const sf_config* cfg, sf_engine** out);
/* Synchronises the device and frees the engine.  Streams still alive are
 * detached: sf_stream_destroy still frees them (and sf_stream_reset and
 * sf_stream_window still work), every other call on them returns SF_EINVAL. */
SF_API sf_status sf_destroy(sf_engine* e);
SF_API sf_status sf_get_metadata(const sf_engine* e, sf_config* out);
/* Message of the last error on this engine (never NULL; "" if none). */
SF_API const char* sf_last_error(const sf_engine* e);
SF_API const char* sf_status_str(sf_status s);

/* ------------------------------------------------------------ front-end */

/* Preprocessor ("Exported Methods / preprocessor": audio (N,) + length ->
 * mel (1, 128, T) + mel_len), batched.
 *   d_audio  f32 [B x n_max]  16 kHz mono, clip b valid for h_len[b] samples
 *   h_len    i64 [B]          1600 <= h_len[b] <= min(n_max, max_samples)
 *   d_mel    f32 [B x 128 x (1 + n_max/160)]  normalised log-mel; every
 *            element is written, frames >= h_mel_len[b] are 0
 *   h_mel_len i64 [B] (out)   h_len[b] / 160
 * Preemphasis 0.97, centred STFT (n_fft 512, Hann 400, hop 160), power,
 * 128 Slaney mel bins 0-8 kHz, log(x + 2^-24), per-bin mean/std
 * normalisation over the valid frames. */
SF_API sf_status sf_mel(sf_engine* e, const float* d_audio, const int64_t* h_len, int B, int64_t n_max,
                 float* d_mel, int64_t* h_mel_len, void* cuda_stream);

/* Allocation-free front-end.  The pages have no counterpart to this call: it
 * exists for callers that cannot allocate device memory when they compute
 * features (a pre-budgeted memory pool they do not own, a plugin inside
 * another framework's CUDA context, a real-time thread that must not block
 * in cudaMalloc/cudaFree).  Same arguments, layout and result as sf_mel, but
 * no engine is needed and nothing is allocated: the call's scratch (clip
 * lengths, per-tile statistics and per-clip normalisation constants) is a
 * fixed static device array of about 8 MiB in libsf.so that every GPU
 * loading the library keeps until exit.
 * Limits: B <= 64 clips and B * ceil((1 + n_max/160) / 32) <= 4096 frame
 * tiles (e.g. 10 clips of 120 s); larger requests return SF_ESHAPE.
 * The first call on a device (with that device current) takes the array's
 * device address, uploads the FFT/window/filterbank tables with a blocking
 * copy and sets the frame kernels' shared-memory attribute for the device.
 * All calls share the array and it keeps the last
 * call's contents, so calls whose GPU work overlaps (on different streams or
 * threads) race and corrupt each other; order them on one stream.  No error
 * message is kept (there is no engine): the status code is the report. */
SF_API sf_status sf_mel_noalloc(const float* d_audio, const int64_t* h_len, int B, int64_t n_max, float* d_mel,
                                int64_t* h_mel_len, void* cuda_stream);

/* ------------------------------------------------- exported-method split */

/* pre_encode ("Exported Methods / pre_encode": chunk (1, T, 128) -> embs
 * (1, 1+(T-1)//8, 512)), batched over windows of normalised features.
 *   d_feats  f32 [n_buf x 128 x t_buf]  channels-first features
 *   h_buf    i32 [n]  which buffer row each window reads
 *   h_start  i64 [n]  first column of the window in that row
 *   h_frames i64 [n]  window length W_i (>= 1); columns outside
 *                     [start, start + W_i) are treated as zero
 *   d_embs   act [n x emb_stride x d_model] (out) window i's
 *            1 + (W_i-1)//8 embeddings; emb_stride >= the largest count */
SF_API sf_status sf_pre_encode(sf_engine* e, const float* d_feats, int n_buf, int64_t t_buf, const int* h_buf,
                        const int64_t* h_start, const int64_t* h_frames, int n, void* d_embs,
                        int64_t emb_stride, void* cuda_stream);

/* encode ("Exported Methods / encode": embs (1, T_total, 512) -> preds
 * (1, T_total, 4)), over n packed sequences.
 *   d_embs   act [sum(h_seq_len) x d_model]  sequences back to back
 *   h_seq_len i32 [n]  each >= 1, <= the longest sequence supported
 *   d_preds  f32 [sum(h_seq_len) x n_spk] (out) sigmoid probabilities */
SF_API sf_status sf_encode(sf_engine* e, const void* d_embs, const int* h_seq_len, int n, float* d_preds,
                    void* cuda_stream);

/* ----------------------------------------------------------------- offline */

/* forward(audio, lengths) -> probs (NeMo Speaker Diarization API, forward).
 *   d_audio, h_len, B, n_max as for sf_mel
 *   d_probs   f32 [B x T'_max x 4] (out), T'_max = 1 + (n_max/160 - 1)/8;
 *             rows >= h_out_len[b] are 0
 *   h_out_len i64 [B] (out) = 1 + (h_len[b]/160 - 1)/8 */
SF_API sf_status sf_forward_offline(sf_engine* e, const float* d_audio, const int64_t* h_len, int B, int64_t n_max,
                             float* d_probs, int64_t* h_out_len, void* cuda_stream);

/* Same, from and to HOST memory (pinned or pageable): the call copies the
 * audio to the device, runs, copies the probabilities back and
 * synchronises on `cuda_stream`. */
SF_API sf_status sf_forward_offline_host(sf_engine* e, const float* h_audio, const int64_t* h_len, int B,
                                  int64_t n_max, float* h_probs, int64_t* h_out_len, void* cuda_stream);

/* ---------------------------------------------------------------- streaming */

/* A batch of n_streams independent streams sharing one preset; all state
 * (cache, FIFO, predictions, silence mean) lives on the device. */
SF_API sf_status sf_stream_create(sf_engine* e, const sf_preset* p, int n_streams, sf_stream** out);
/* Synchronises the device, frees the stream's state and the engine's CUDA
 * graphs that were captured for it. */
SF_API sf_status sf_stream_destroy(sf_stream* s);

/* Restore the empty state of the listed streams (h_ids NULL = all; else
 * n >= 0 ids in [0, n_streams), SF_EINVAL otherwise).  Synchronises the
 * device before and after clearing the device-side silence statistics, so
 * it is ordered against steps on any CUDA stream. */
SF_API sf_status sf_stream_reset(sf_stream* s, const int* h_ids, int n);

/* Mel-frame window [*h_start, *h_end) the next step of stream `id` reads
 * for a recording of h_total valid mel frames: one encoder frame (8 mel
 * frames) of left context when the stream is past its first chunk, then
 * chunk_len + right_context encoder frames, clipped at the end. */
SF_API sf_status sf_stream_window(const sf_stream* s, int id, int64_t h_total, int64_t* h_start, int64_t* h_end);

/* One step of every unfinished stream (forward_streaming_step):
 * pre_encode on the new window only, encoder on [cache | FIFO | chunk],
 * chunk predictions out (look-ahead frames are attended to but not
 * emitted), FIFO push/pop, cache compression.
 *   d_feats      f32 [n_streams x 128 x t_buf] normalised features; column t
 *                of stream i is mel frame h_feat_start[i] + t
 *   h_feat_start i64 [n_streams]
 *   h_feat_end   i64 [n_streams]  the recording has h_feat_end[i] mel
 *                frames (a window reaching past it is clipped there; a
 *                step whose window reaches it finishes the stream)
 *   d_chunk_probs f32 [n_streams x chunk_len x 4] (out); rows >= h_n_out[i] are 0
 *   h_n_out      i32 [n_streams] (out) frames emitted (0 for finished streams)
 * The window columns the step needs must lie inside the buffer (SF_ESHAPE). */
SF_API sf_status sf_stream_step(sf_stream* s, const float* d_feats, int64_t t_buf, const int64_t* h_feat_start,
                         const int64_t* h_feat_end, float* d_chunk_probs, int* h_n_out, void* cuda_stream);

/* Audio-in streaming step: the step computes each stream's mel window
 * itself from raw audio instead of taking features.  Reading (the HF
 * streaming notes slice the audio per chunk and run the processor on each
 * slice, without saying how features are normalised; the NeMo API streams
 * features normalised over the whole clip): the window's frames m0 .. m1-1
 * are the centred frames of the stream's continuous signal (preemphasis and
 * STFT exactly as sf_mel, zeros past the audio received so far), normalised
 * per bin over the window's own frames (same formula as sf_mel over a clip).
 *   d_audio        f32 [n_streams][n_buf]  row = stream; column 0 holds sample
 *                  h_audio_start[id] of that stream, h_audio_end[id] samples
 *                  (absolute) have arrived
 *   h_final        i32 [n_streams]  1 once the stream's audio has ended
 * A stream steps when its window is complete: its last frame (chunk plus
 * right context) has all its samples, i.e. audio_end >= 160 x (8 x (c0 +
 * chunk_len + right_context)) + 96 with c0 the next encoder frame; a final
 * stream steps with what it has and finishes after its last frame.  Other
 * streams emit 0 frames; a call where no stream is ready does nothing and
 * returns SF_OK.  The buffer row must start no later than sample
 * 160 x m0 - 257 of the window (m0 = 8 x (c0 - 1), 0 for the first step).
 * Outputs as sf_stream_step. */
SF_API sf_status sf_stream_step_audio(sf_stream* s, const float* d_audio, int64_t n_buf,
                                      const int64_t* h_audio_start, const int64_t* h_audio_end, const int* h_final,
                                      float* d_chunk_probs, int* h_n_out, void* cuda_stream);

/* Copy one stream's state out to / in from caller buffers (forward_for_export
 * style state injection).  Synchronise on `cuda_stream`. */
SF_API sf_status sf_stream_get_state(sf_stream* s, int id, sf_state_view* v, void* cuda_stream);
SF_API sf_status sf_stream_set_state(sf_stream* s, int id, const sf_state_view* v, void* cuda_stream);

/* State update alone (FIFO refresh/push/pop, silence mean, compression)
 * given each stream's window predictions, for teacher-forced checks of the
 * bookkeeping.  Stream i's window is [cache | FIFO | n_new[i] new frames].
 *   d_preds    f32 [sum_i (n_cache_i + n_fifo_i + h_n_new[i]) x 4] packed
 *   d_new_embs act [n_streams x new_stride x d_model] new frames' embeddings
 *   h_n_new    i32 [n_streams] new frames (chunk + look-ahead), 0 = skip stream
 *   d_scores   f32 [n_streams x (spkcache_len + fifo_len + chunk_len) x 4]
 *              (out, may be NULL) compression scores, -inf = not a candidate
 *   d_src      i32 [n_streams x spkcache_len] (out, may be NULL) source of each
 *              new cache slot after a compression: candidate index, or
 *              -1 - s for a placeholder of speaker s; untouched otherwise
 *   d_scores_in f32, same shape as d_scores, or NULL: use these scores
 *              instead of computing them */
SF_API sf_status sf_stream_update(sf_stream* s, const float* d_preds, const void* d_new_embs, int64_t new_stride,
                           const int* h_n_new, float* d_scores, int* d_src, const float* d_scores_in,
                           void* cuda_stream);

/* Per-speaker top-k selection alone (the compression's selection step).
 *   d_scores f32 [n_sets x stride x n_spk], set i has h_n[i] candidates
 *   d_src    i32 [n_sets x (k * n_spk)] (out) kept candidate indices in
 *            ascending order, then -1 - s placeholders in speaker order
 * Order: score descending, candidate index ascending; -inf never kept. */
SF_API sf_status sf_select_topk(sf_engine* e, const float* d_scores, const int* h_n, int n_sets, int stride, int k,
                         int* d_src, void* cuda_stream);

/* ----------------------------------------------------------- segments */

/* Post-processing of frame probabilities into speaker segments ("Streaming
 * Sortformer Diarizer" model card, Output: diarize() turns the (B, T/8, 4)
 * sigmoid probabilities into [start_seconds, end_seconds, speaker_index]
 * segments by VAD-style thresholding and smoothing; NeMo API page,
 * SortformerEncLabelModel.diarize).  Per clip and speaker, in this order:
 *   1. hysteresis: a run starts at a frame with p > onset and ends before the
 *      first later frame with p <= offset (onset = offset: active <=> p > it);
 *   2. a run of encoder frames a..b covers [0.08 a, 0.08 (b + 1)) seconds;
 *   3. padding: start - pad_onset (>= 0), end + pad_offset (<= 0.08 n_frames);
 *   4. a segment joins the previous one when it starts at or before its end
 *      or less than min_duration_off after it;
 *   5. merged segments shorter than min_duration_on are dropped.
 * Times are float64 with each product and sum rounded separately. */
typedef struct sf_seg_params {
  float onset, offset;                       /* onset >= offset, both in [0, 1] */
  double pad_onset, pad_offset;              /* seconds, >= 0 */
  double min_duration_on, min_duration_off;  /* seconds, >= 0 */
} sf_seg_params;

/* Defaults: onset = offset = 0.5, no padding, no duration limits. */
SF_API sf_status sf_default_seg_params(sf_seg_params* out);

/*   d_probs    f32 [n][stride_t][4]  per-clip probabilities (sf_forward_offline's
 *                                    output layout, or chunk outputs gathered by
 *                                    the caller)
 *   h_n_frames i32 [n] host          frames of each clip, 0 <= n_frames <= stride_t
 *   d_segs     f64 [n][4][max_seg][2] (out)  start, end seconds, in time order
 *   d_counts   i32 [n][4] (out)      segments found per clip and speaker; may
 *                                    exceed max_seg, only the first max_seg
 *                                    are stored
 * 1 <= n <= 512.  Device buffers are the caller's; the
 * engine's descriptor block carries the frame counts (ordered on
 * `cuda_stream` with the engine's other calls). */
SF_API sf_status sf_segments(sf_engine* e, const float* d_probs, int stride_t, const int* h_n_frames, int n,
                             const sf_seg_params* params, int max_seg, double* d_segs, int* d_counts,
                             void* cuda_stream);

/* ---------------------------------------------------------------- options */

enum {
  SF_OPT_GRAPHS = 1,     /* 1 (default): capture each call shape once as a CUDA graph and
                            replay it; 0: launch kernel by kernel */
  SF_OPT_PDL = 2,        /* 1 (default): programmatic dependent launch between kernels (each
                            kernel may start its set-up and weight loads while its predecessor
                            finishes; single-wave GEMMs then use half the operand ring so two
                            CTAs share an SM); 0 plain stream order (same results to the bit) */
  SF_OPT_GEMM_PATH = 3,  /* bf16 projections on the tcgen05/TMEM/TMA kernels: 1 (default) with
                            multi-wave projections of K >= 1024 and width >= 256 on CTA
                            pairs (tcgen05 cta_group::2, 256-row tiles), 2 every multi-wave
                            projection on CTA pairs, 3 single CTAs only; 0 the mma.sync
                            kernel */
  SF_OPT_GEMM_PAIR_BN = 4, /* tile width of the CTA-pair kernel: 0 (default) chosen per shape,
                              or 128, 192, 256 */
  SF_OPT_ATTN_PATH = 5,   /* bf16 attention (relative-position and Transformer): 1 (default)
                             tcgen05/TMEM/TMA kernels, whose keys are split over CTA clusters
                             when one sequence leaves SMs idle; 0 mma.sync kernels */
  SF_OPT_MEL_PATH = 6,    /* log-mel front-end (sf_mel, the offline forward, the audio-in
                             step): 1 (default) FFT in registers with warp shuffles, then
                             separate statistics and normalisation passes over all SMs; 0 FFT
                             through shared memory and one normalisation CTA per (clip, bin) */
  SF_OPT_LN_FUSE = 8,     /* bf16 engines: 1 (default) LayerNorm fused into the epilogue of the
                             residual projection before it wherever the projection's 64-column
                             tiles of a 128-row block fit one CTA cluster and all row blocks
                             one wave; 0 separate LayerNorm kernels */
  SF_OPT_TF_FUSE = 9,     /* bf16 engines, Transformer layers: 1 (default) everything after each
                             layer's attention (output projection, LN1, FFN, LN2 and the next
                             layer's Q|K|V projection) in one kernel per layer, a cluster of four
                             CTAs per 128-row block, when one wave of clusters covers the rows; 2
                             that kernel for any number of rows; 0 separate projections */
  SF_OPT_SUB_PATH = 7     /* ConvSubsampling's first two stages: 1 (default) one kernel that
                             computes the first conv's outputs on chip and feeds them straight
                             into the first depthwise conv; 0 the 3x3 s2 conv and the first
                             depthwise conv as two kernels through a [T/2][64][256] tensor in
                             memory (same result to the bit) */
};
SF_API sf_status sf_set_option(sf_engine* e, int option, int value);

/* ------------------------------------------------------------ diagnostics */

/* Synchronise `cuda_stream` and read (then clear) the engine's device error
 * word: SF_ETIMEOUT if a kernel's bounded wait gave up, SF_EDEVICE if a
 * device-side index check skipped an access, SF_OK otherwise. */
SF_API sf_status sf_check(sf_engine* e, void* cuda_stream);

/* Failure-detection self-test: enqueue one kernel that waits, through the
 * bounded device wait every tcgen05 kernel uses, on a barrier that nothing
 * completes.  The wait gives up after its clock budget (about 2 s), records
 * the timeout in the engine's error word and returns; the next sf_check
 * returns SF_ETIMEOUT (and clears the word), and the engine and the CUDA
 * context remain usable.  Errors: SF_EINVAL, SF_ECUDA (launch). */
SF_API sf_status sf_selftest_wait(sf_engine* e, void* cuda_stream);

/* The engine's dense projection alone, for tests and kernel benchmarks:
 *   d_C [M x N] (out) = d_A bf16 [M x K] (row stride lda) .
 *       d_W bf16 [N x K]^T + d_bias f32 [N] (may be NULL)
 * path 1 = tcgen05/TMEM/TMA kernel (the engine's), 0 = mma.sync kernel,
 * both writing f32 C.  The engine's fused epilogues on the tcgen05 kernel:
 * path 2 = bf16 C; 3 = residual update, f32 C [M x N] += result; 4 = bf16
 * C = swish(result); 5 = gated linear unit, bf16 C [M x N/2] with
 * C[:, j] = r[:, 2j] * sigmoid(r[:, 2j + 1]) (value/gate columns interleaved).
 * Requires N % 16 == 0, K % 64 == 0, lda % 8 == 0, 16-byte aligned A/W. */
SF_API sf_status sf_gemm_bf16(sf_engine* e, const void* d_A, int lda, const void* d_W, int M, int N, int K,
                              const float* d_bias, void* d_C, int path, void* cuda_stream);

/* The engine's residual projection with the LayerNorm that follows it fused
 * into the epilogue (bf16 engines), for tests and kernel benchmarks; the
 * conformer and Transformer layers' "x = x + f(x); h = LN(x)" steps
 * ("Streaming Sortformer Diarizer", Pipeline: FastConformer and post-LN
 * Transformer layers):
 *   x_new = d_x f32 [M x N] + alpha (d_A bf16 [M x K] . d_W bf16 [N x K]^T
 *           + d_bias f32 [N] (may be NULL))
 *   xnorm 0: d_x <- x_new,     d_h bf16 [M x N] <- LN(x_new)
 *   xnorm 1: d_x <- LN(x_new), d_h <- LN2(LN(x_new)) with d_g2/d_b2, else LN(x_new)
 * LN(v) = (v - mean) / sqrt(var + 1e-5) * g + b over each row (biased
 * variance), g/b f32 [N].  Requires N a multiple of 64 up to 512 and every
 * 128-row block's cluster of N/64 CTAs co-resident (SF_ESHAPE otherwise),
 * K % 64 == 0, lda % 8 == 0, 16-byte aligned A/W/x/h. */
SF_API sf_status sf_gemm_bf16_ln(sf_engine* e, const void* d_A, int lda, const void* d_W, int M, int N, int K,
                                 const float* d_bias, float alpha, float* d_x, const float* d_g, const float* d_b,
                                 const float* d_g2, const float* d_b2, int xnorm, void* d_h, void* cuda_stream);

/* The engine's relative-position self-attention alone (bf16 engines), for
 * tests and kernel benchmarks ("Streaming Sortformer Diarizer" model card,
 * FastConformer encoder: relative-position MHSA, d_model 512, 8 heads of 64):
 *   d_qkv  bf16 [M x 1536]  rows of the n packed sequences (h_seq_len[i]
 *                           rows each, M = their sum), columns q | k | v,
 *                           head h at columns 64h .. 64h + 63 of each part
 *   d_ptab bf16 [(2R-1) x 512]  projected relative-position rows; row
 *                           i - j + R - 1 holds distance i - j
 *   d_u, d_v f32 [512]      per-head position biases (pos_bias_u / _v)
 *   d_ctx  bf16 [M x 512] (out)  softmax_j(((q_i+u).k_j + (q_i+v).p_(i-j))/8) v_j
 * Sequence lengths must lie in [1, R]; path 1 = tcgen05 kernel, 0 = mma.sync.
 * Pointers 16-byte aligned.  Uses the engine's descriptor block (ordered on
 * `cuda_stream` with the engine's other calls). */
SF_API sf_status sf_attention_relpos(sf_engine* e, const void* d_qkv, const void* d_ptab, int R, const float* d_u,
                                     const float* d_v, const int* h_seq_len, int n, void* d_ctx, int path,
                                     void* cuda_stream);

/* The Transformer encoder's self-attention alone (bf16 engines), for tests
 * and kernel benchmarks ("Streaming Sortformer Diarizer" model card: 18-layer
 * Transformer, d_model 192, 8 heads of 24):
 *   d_qkv bf16 [M x 576]  rows of the n packed sequences (h_seq_len[i] rows
 *                         each), columns q | k | v, head h at columns
 *                         24h .. 24h + 23 of each part
 *   d_ctx bf16 [M x 192] (out)  softmax_j(q_i . k_j / sqrt(24)) v_j
 * Sequence lengths in [1, the engine's longest sequence]; path 1 = tcgen05
 * kernel (keys split over CTA clusters when the (query tile, head) units
 * leave SMs idle), 0 = mma.sync.  Pointers 16-byte aligned.  Uses the engine's
 * descriptor block (ordered on `cuda_stream` with its other calls). */
SF_API sf_status sf_attention_mha(sf_engine* e, const void* d_qkv, const int* h_seq_len, int n, void* d_ctx, int path,
                                  void* cuda_stream);

/* ---------------------------------------------------------------- profiling */

/* Per kernel class: launches, device time between CUDA events recorded on
 * the launching stream around each launch, and the algorithmic work of those
 * launches (flops of the contraction, or the bytes the operation must move
 * through HBM at minimum). */
typedef struct {
  char name[32];
  int64_t launches;
  double ms;
  double flops;
  double bytes;
} sf_kernel_stat;

/* Launch counting is always on.  enable = 1 also brackets every launch with
 * a pair of CUDA events (each pair adds a few microseconds; use for
 * attribution, not for end-to-end timing); enable = 2 * mask brackets only
 * the kernel classes whose bit is set in `mask` (bit k = the k-th class in
 * the order mel, conv1, dwconv3x3s2, gemm, attention_relpos, attention_mha,
 * layernorm, dwconv1d, head_out, assemble, extract, state_update, to_f32,
 * select_topk, tf_layer); enable = 0 stops recording. */
SF_API sf_status sf_profile_enable(sf_engine* e, int enable);
/* Synchronise on the recorded events and report one entry per kernel class
 * with at least one launch since the last reset (at most `max` entries,
 * count in *n_out).  reset = 1 clears the counters afterwards. */
SF_API sf_status sf_profile_read(sf_engine* e, sf_kernel_stat* out, int max, int* n_out, int reset);

/* ------------------------------------------------ Nemotron-3 variant (offline) */

/* The Nemotron-3 diarization model's offline forward ("Enable
 * Nemotron-3-Diarization on MLX, CUDA, XNNPACK, and Vulkan", model
 * description: 16 kHz mono audio, 128-bin mel stacked to 80 ms encoder
 * frames, a 31-layer Transformer with rotary position embedding, a Conv1D
 * upsampling head giving up to 8 speakers' activity every 10 ms;
 * Transformers "Nemotron 3 Diarization": logits (1, frames, 8), one frame
 * every 10 ms).  The pages give no widths; this engine implements the
 * readings d_model 512 in 8 heads of 64, FFN 2048 (swish), pre-LN layers and
 * a final LayerNorm, frame-major stacking of 8 normalised mel frames into a
 * Linear 1024 -> 512, rotate-half RoPE from each clip's start (base 10000),
 * and a transposed conv with kernel = stride = 8 (512 -> 8 speakers) and a
 * sigmoid as the head.  bf16 weights and activations, fp32 accumulation and
 * residual stream.  Streaming (the arrival-order speaker cache) is not
 * implemented here. */
typedef struct sf_nem_engine sf_nem_engine;
typedef struct {
  int n_layers;          /* Transformer layers (31; any count >= 1)                  */
  int d_model;           /* must be 512                                              */
  int ff;                /* must be 2048                                             */
  int n_spk;             /* must be 8                                                */
  int max_batch;         /* clips per call, 1 .. 512                                 */
  int64_t max_samples;   /* longest clip, 1,600 .. 230,400,000 samples               */
} sf_nem_config;
SF_API sf_status sf_nem_default_config(sf_nem_config* out);
/* Weights: the SFW1 container with tensors nem.stack.weight [512 x 1024],
 * nem.stack.bias [512], per layer l nem.layers.l.{ln1,ln2}.{weight,bias}
 * [512], .att.{q,k,v,o}.weight [512 x 512] and .bias [512],
 * .ff.linear1.weight [2048 x 512], .ff.linear1.bias [2048],
 * .ff.linear2.weight [512 x 2048], .ff.linear2.bias [512], then
 * nem.final_ln.{weight,bias} [512], nem.head.weight [512 x 8 x 8]
 * (in channel, speaker, tap), nem.head.bias [8].  Copies and converts the
 * weights, allocates the workspace for max_batch clips of max_samples and
 * synchronises.  Errors: SF_EINVAL (configuration), SF_EDEVICE (not an
 * sm_100 device), SF_EFORMAT, SF_ENOMEM, SF_ECUDA. */
SF_API sf_status sf_nem_create(const void* h_blob, uint64_t nbytes, const sf_nem_config* cfg, sf_nem_engine** out);
/* Synchronises the device and frees the engine. */
SF_API sf_status sf_nem_destroy(sf_nem_engine* e);
/* Offline forward of B clips:
 *   d_audio   f32 [B x n_max]  16 kHz mono, clip b's first h_len[b] samples valid
 *   h_len     i64 [B]  each in [1600, n_max]
 *   d_probs   f32 [B x (n_max / 160) x 8] (out)  speaker activity every 10 ms;
 *             frames at or past a clip's h_len / 160 are written as 0
 *   h_out_len i64 [B] (out, may be NULL)  h_len / 160
 * Synchronises on cuda_stream (reads the device error word).  Errors:
 * SF_EINVAL, SF_ESHAPE (B or n_max beyond the configuration), SF_EDEVICE
 * (another device is current), SF_ETIMEOUT (a bounded device wait gave up),
 * SF_ECUDA. */
SF_API sf_status sf_nem_forward_offline(sf_nem_engine* e, const float* d_audio, const int64_t* h_len, int B,
                                        int64_t n_max, float* d_probs, int64_t* h_out_len, void* cuda_stream);
SF_API const char* sf_nem_last_error(const sf_nem_engine* e);

#ifdef __cplusplus
}
#endif
#endif /* SF_H_ */
