/*
 * dmel.h — C ABI of the dMel audio front end on NVIDIA B200 (sm_100a).
 *
 * The front end turns 16 kHz mono waveforms into one D-dimensional vector per 50 ms frame
 * ("Inside Inkling: Audio Design", Part 1 · Modeling): 1600-sample windows at an 800-sample
 * hop, power spectrum, 80 mel channels, log, clamp to [-7, 2], 16 levels per channel, then the
 * sum of the 80 table rows 16*b + c_b of a 1280 x D embedding table with an optional RMSNorm.
 * The readings of what the pages leave open (causal framing, periodic Hann window, 1600-point
 * DFT, HTK mel triangles, log10 with a 1e-10 floor, 16 equal levels, row layout) are stated at
 * each entry point below.
 *
 * Conventions for every call
 *   - Pointers named h_* are host memory; every other array pointer is device memory of the
 *     current CUDA device. The caller allocates and owns all of them; the library keeps no
 *     pointer after a call returns.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default stream) and
 *     never synchronise, except that the first call on each device uploads constant tables
 *     (window, twiddles, mel weights) with a blocking copy; make that first call before any
 *     stream capture.
 *   - Arguments are checked on the host before anything is launched; a bad argument returns
 *     DMEL_ERR_INVALID_ARG and launches nothing. A failed launch returns DMEL_ERR_CUDA.
 *     Device-side faults are never used as error reports: kernels that find bad data (a code
 *     above 15, an offset that does not match) record it in a device error word that
 *     dmel_get_device_error() reads, and carry on with a clamped value.
 *   - n_clips == 0 or n_frames == 0 is a valid call that does nothing.
 *   - No entry point allocates device memory. Scratch space comes from the caller's workspace;
 *     dmel_workspace_size() says how much. The one exception is dmel_embed_noalloc, whose
 *     scratch is a fixed array inside the library (see there); dmel_forward_host also creates
 *     two copy streams per device on its first call.
 *   - Calls may come from several host threads at once (each with its own buffers): the
 *     per-device one-time setup (constant tables, kernel attributes) is guarded, and
 *     dmel_last_launch_count() reports the calling thread's last call.
 *   - Environment (read once per process): DMEL_EMBED_MMA=dense runs the tensor-core embedding
 *     as a dense one-hot product instead of the 2:4-sparse one; DMEL_EMBED_TILE=single runs it
 *     dense on one-CTA tiles instead of CTA pairs; DMEL_COOPERATIVE=0 launches the fused
 *     RMSNorm kernels without the cooperative attribute (for profilers that cannot replay
 *     cooperative cluster launches). All exist for comparison and measurement.
 */
#ifndef DMEL_H
#define DMEL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;
typedef struct CUstream_st *dmel_stream_t; /* same object as cudaStream_t */

typedef enum {
  DMEL_OK = 0,
  DMEL_ERR_INVALID_ARG = 1, /* a pointer, size, offset or flag is out of contract */
  DMEL_ERR_UNSUPPORTED = 2, /* valid request that this build does not run (e.g. no sm_100 device) */
  DMEL_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  DMEL_ERR_TOO_LARGE = 4    /* dmel_embed_noalloc: the request needs more than its fixed scratch */
} dmel_status;

typedef enum { DMEL_F32 = 0, DMEL_BF16 = 1 } dmel_dtype;

#define DMEL_SAMPLE_RATE 16000
#define DMEL_HOP 800        /* 50 ms: 20 frames per second */
#define DMEL_WIN 1600       /* 100 ms window, also the DFT size */
#define DMEL_N_BINS 801     /* one-sided DFT bins, 10 Hz apart */
#define DMEL_N_MEL 80       /* mel channels */
#define DMEL_N_LEVELS 16    /* quantisation levels per channel */
#define DMEL_TABLE_ROWS 1280 /* 80 x 16 */
#define DMEL_MODEL_DIM 6144 /* embedding width of the released model */

/* Device error word bits (see dmel_get_device_error). */
#define DMEL_DEVERR_CODE_RANGE 0x1u  /* a code above 15 reached an embedding kernel (used code & 15) */
#define DMEL_DEVERR_WAIT_TIMEOUT 0x2u /* a pipeline wait inside a kernel gave up (results invalid) */
#define DMEL_DEVERR_OFFSETS 0x4u     /* device frame offsets disagree with the sample offsets */
#define DMEL_DEVERR_OUT_ROW 0x8u     /* an output row index outside [0, out_n_rows) (row not written) */

/* Frames of one clip of n_samples samples: floor(n_samples / 800) (20 per second of audio;
 * "Inside Inkling: Audio Design", Part 1 · Modeling). Host only, pure. Returns -1 for
 * n_samples < 0. */
int64_t dmel_frames_for_length(int64_t n_samples);

/* Host exclusive scan of frame counts: h_frame_offsets[0] = 0,
 * h_frame_offsets[c+1] = h_frame_offsets[c] + dmel_frames_for_length(len_c), where
 * len_c = h_sample_offsets[c+1] - h_sample_offsets[c]. Both arrays have n_clips + 1 entries.
 * This is the per-item frame count the serving renderer reports as "audio_tokens"
 * ("Inside Inkling: Audio Design", Part 3 · Inference). Errors: DMEL_ERR_INVALID_ARG when a
 * pointer is NULL, n_clips < 0, h_sample_offsets[0] != 0 or the offsets decrease. */
dmel_status dmel_frame_offsets(const int64_t *h_sample_offsets, int n_clips, int64_t *h_frame_offsets);

/* Bytes of device workspace that dmel_embed / dmel_forward need for this request (0 when none).
 * with_codes_out: nonzero when the caller passes its own codes buffer to dmel_forward.
 * with_rmsnorm: nonzero when rms_weight will be non-NULL. */
size_t dmel_workspace_size(int64_t n_frames, int embed_dim, dmel_dtype table_dtype, int with_rmsnorm,
                           int with_codes_out);

/* dMel codes of every frame of a batch of clips.
 *
 * wav             fp32 samples of all clips, concatenated with no padding [sample_offsets[n_clips]]
 * sample_offsets  int64 [n_clips + 1], device copy of the host offsets (start 0, non-decreasing)
 * frame_offsets   int64 [n_clips + 1], device copy of dmel_frame_offsets() of the same offsets
 * n_clips         number of clips (>= 0)
 * n_frames        h_frame_offsets[n_clips] (host value, so no device read is needed to size the grid)
 * tails           NULL, or fp32 [n_clips x 800]: the 800 samples that came before each clip
 *                 (streaming); NULL means zeros
 * tails_out       NULL, or fp32 [n_clips x 800]: receives the 800 samples that end at sample
 *                 800*F of each clip (F its frame count), or the tail in when F == 0. Must not
 *                 overlap wav. May equal `tails`: it is then written by a kernel of its own after
 *                 every frame has been read; a tails_out apart from `tails` (two buffers used in
 *                 turn, for streaming) is written by the codes kernel itself, one launch fewer.
 * codes           uint8 [n_frames x 80], row-major, receives c_b in 0..15 per frame and channel
 *
 * Per frame t of a clip x (causal framing, "Inside Inkling: Audio Design", Part 1 · Modeling:
 * hop 800, window 1600): s[n] = x[800 (t-1) + n], n < 1600, samples before the clip from the
 * tail; P_k = |sum_n w[n] s[n] e^{-2 pi i k n/1600}|^2 with w the periodic Hann window;
 * M_b = sum_k H_b(10 k Hz) P_k with 80 HTK mel triangles on 0..8000 Hz;
 * L = min(max(log10(max(M_b, 1e-10)), -7), 2); c_b = min(15, floor((L + 7) * 16 / 9)).
 * The DFT runs in fp64; the mel sums, log10, clamp and quantiser run in fp32 (they move L by
 * ~1e-7 at most). Errors: DMEL_ERR_INVALID_ARG for NULL required pointers, n_clips < 0 or
 * n_frames < 0. */
dmel_status dmel_codes(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                       int64_t n_frames, const float *tails, float *tails_out, uint8_t *codes, dmel_stream_t stream);

/* Embedding of dMel codes ("Inside Inkling: Audio Design", Part 1 · Modeling: each
 * (channel, level) pair owns one row; a frame's 80 rows are summed; optional RMSNorm).
 *
 * codes        uint8 [n_frames x 80], values 0..15 (a larger value is used as value & 15 and
 *              flagged in the device error word)
 * table        [1280 x embed_dim] row-major, fp32 or bf16 (table_dtype); row of channel b and
 *              level c is 16 b + c
 * embed_dim    D, a positive multiple of 8 (6144 for the model). bf16 tables with D a multiple
 *              of 256 run on the tensor cores (tcgen05); other requests run on the CUDA cores,
 *              which take D <= 16384.
 * rms_weight   NULL (no RMSNorm) or [embed_dim] in table_dtype: y_j = g_j x_j / sqrt(mean x^2 + eps)
 * eps          RMSNorm epsilon (> 0 when rms_weight is given; the model uses 1e-6)
 * out          [n_frames x embed_dim] in out_dtype (fp32, or bf16 rounded to nearest even)
 * workspace    device scratch of at least dmel_workspace_size(n_frames, embed_dim, table_dtype,
 *              rms_weight != NULL, 1) bytes, 256-byte aligned (may be NULL when that size is 0)
 * Sums accumulate in fp32. */
dmel_status dmel_embed(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype, int embed_dim,
                       const void *rms_weight, float eps, void *out, dmel_dtype out_dtype, void *workspace,
                       size_t workspace_bytes, dmel_stream_t stream);

/* dmel_embed for callers that cannot allocate device memory: the paper has no counterpart of
 * this entry point; it exists for integration only.
 *
 * Some callers have no way to provide a workspace: a real-time audio callback or a serving
 * step being captured into a CUDA graph may not call cudaMalloc (it can synchronise the device
 * and is not allowed during stream capture), and some host frameworks own all device memory
 * and hand a library nothing but input and output pointers. This variant takes the same
 * arguments as dmel_embed minus the workspace and allocates nothing: the scratch it needs (the
 * RMSNorm partial sums of the tensor-core path) is a fixed 4 MiB array inside the library,
 * which every device that loads the library holds until the process exits.
 *
 * Limit: with rms_weight != NULL and a bf16 table whose embed_dim is a multiple of 256, the
 * request needs the scratch dmel_workspace_size(n_frames, embed_dim, DMEL_BF16, 1, 1) reports,
 * about n_frames * ceil(embed_dim / 192) * 4 bytes (up to 32,640 frames at embed_dim 6144); a
 * larger request returns DMEL_ERR_TOO_LARGE and launches nothing. Other requests need no
 * scratch and have no extra limit.
 *
 * The first call on each device looks up the scratch's device address (and uploads nothing
 * else); make that first call before any stream capture. All calls share the one scratch
 * array, which keeps the last call's contents (every value a call reads it writes first):
 * calls that overlap on the GPU, e.g. on two streams at once, race on it and must be ordered
 * by the caller. */
dmel_status dmel_embed_noalloc(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                               int embed_dim, const void *rms_weight, float eps, void *out, dmel_dtype out_dtype,
                               dmel_stream_t stream);

/* dmel_codes followed by dmel_embed on the same stream: waveforms to frame vectors.
 * Arguments are those of the two calls; codes_out is NULL (codes kept in the workspace) or
 * uint8 [n_frames x 80] to receive the codes as well. workspace must hold
 * dmel_workspace_size(n_frames, embed_dim, table_dtype, rms_weight != NULL, codes_out != NULL)
 * bytes. */
dmel_status dmel_forward(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                         int64_t n_frames, const float *tails, float *tails_out, const void *table,
                         dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *out,
                         dmel_dtype out_dtype, uint8_t *codes_out, void *workspace, size_t workspace_bytes,
                         dmel_stream_t stream);

/* ---- A table prepared once for many calls. With RMSNorm ("Inside Inkling: Audio Design",
 * Part 1 · Modeling: the summed embedding, optionally normalised), a frame's sum of squares is
 * sum_b sum_b' G[r_b, r_b'] with G = T T^T, the table's Gram matrix (T [1280 x embed_dim], r_b the
 * table row of bin b's level). dmel_embed and dmel_forward compute G inside each call of 16,384
 * frames or more; a caller with a fixed table computes it once here and passes it to the
 * _prepared calls, which then take that form of RMSNorm from 12,288 frames per call (below that,
 * the exchange of row sums inside the product kernel is as fast or faster, and is kept).
 *
 * dmel_table_prepare_size: bytes of the prepared data for a table of this width and dtype, or 0
 *   when no preparation applies (fp32 tables; widths not a multiple of 128).
 * dmel_table_prepare: computes G of table (bf16 [1280 x embed_dim], device, 16-byte aligned) into
 *   prepared (device, 256-byte aligned, prepared_bytes >= dmel_table_prepare_size), owned by the
 *   caller and valid while the table is unchanged. Asynchronous on stream; a size of 0 or a bad
 *   pointer returns DMEL_ERR_INVALID_ARG.
 * dmel_embed_prepared / dmel_forward_prepared: as dmel_embed / dmel_forward, plus prepared (from
 *   dmel_table_prepare for this table, or NULL: then exactly dmel_embed / dmel_forward). It is
 *   used when rms_weight is given and the table qualifies, and ignored otherwise; the workspace
 *   is the one dmel_workspace_size reports. A prepared pointer not 256-byte aligned returns
 *   DMEL_ERR_INVALID_ARG. Results equal the unprepared calls' bit for bit from 16,384 frames
 *   (both take the G form); from 12,288 to 16,383 frames they differ by float rounding only. */
size_t dmel_table_prepare_size(int embed_dim, dmel_dtype table_dtype);
dmel_status dmel_table_prepare(const void *table, int embed_dim, dmel_dtype table_dtype, void *prepared,
                               size_t prepared_bytes, dmel_stream_t stream);
dmel_status dmel_embed_prepared(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                                int embed_dim, const void *rms_weight, float eps, const void *prepared, void *out,
                                dmel_dtype out_dtype, void *workspace, size_t workspace_bytes, dmel_stream_t stream);
dmel_status dmel_forward_prepared(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                                  int n_clips, int64_t n_frames, const float *tails, float *tails_out,
                                  const void *table, dmel_dtype table_dtype, int embed_dim, const void *rms_weight,
                                  float eps, const void *prepared, void *out, dmel_dtype out_dtype,
                                  uint8_t *codes_out, void *workspace, size_t workspace_bytes, dmel_stream_t stream);

/* ---- End to end from host memory: dmel_forward for a batch held in host memory, returning the
 * frame vectors (and optionally the codes) to host memory, with the copies overlapped with the
 * kernels ("Inside Inkling: Audio Design", Part 1 · Modeling for what is computed; Part 3 ·
 * Inference describes featurisation as work done on the host at render time, which is where
 * such batches come from).
 *
 * h_wav             host fp32 samples of all clips, concatenated with no padding
 * h_sample_offsets  host int64 [n_clips + 1] (start 0, non-decreasing)
 * table, table_dtype, embed_dim, rms_weight, eps, out_dtype: as in dmel_embed (device memory)
 * h_out             host [F x embed_dim] in out_dtype, F = the frame count dmel_frame_offsets gives;
 *                   16-byte aligned
 * h_codes           NULL, or host uint8 [F x 80] to receive the codes
 * chunk_frames      frames per pipeline chunk (0: 8192); a chunk may start or end inside a clip
 *                   (its first frame then takes the 800 samples before it from the clip), and the
 *                   results do not depend on it
 * workspace         device scratch of dmel_forward_host_workspace_size(...) bytes with the same
 *                   offsets, widths, types, RMSNorm flag and chunk_frames, 256-byte aligned
 *
 * The frames are cut into chunks; per chunk the samples go to the device on a copy stream of the
 * library's own, the codes and embedding kernels run on `stream`, and the vectors come back on a
 * second copy stream; two device buffer sets alternate, so chunk i + 1 is copied in and chunk
 * i - 1 copied out while chunk i computes. Host buffers should be page-locked (cudaHostAlloc or
 * cudaHostRegister) for the copies to overlap; pageable memory gives the same results, copied
 * synchronously. Asynchronous like every call: the results are in host memory once `stream`
 * reaches the point of the call (cudaStreamSynchronize(stream) waits for them). The host arrays
 * must stay valid and unchanged until then. The first call on a device creates the two copy
 * streams. Errors: DMEL_ERR_INVALID_ARG for bad offsets, a NULL h_wav / h_out with frames to
 * compute, the embedding's argument errors, a negative chunk_frames or a workspace smaller than
 * reported. */
size_t dmel_forward_host_workspace_size(const int64_t *h_sample_offsets, int n_clips, int embed_dim,
                                        dmel_dtype table_dtype, dmel_dtype out_dtype, int with_rmsnorm,
                                        int64_t chunk_frames);
dmel_status dmel_forward_host(const float *h_wav, const int64_t *h_sample_offsets, int n_clips, const void *table,
                              dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *h_out,
                              dmel_dtype out_dtype, uint8_t *h_codes, int64_t chunk_frames, void *workspace,
                              size_t workspace_bytes, dmel_stream_t stream);

/* ---- Quantiser variants. The pages leave the level mapping open ("Inside Inkling: Audio
 * Design", Coda: the quantizer mapping is undocumented, uniform or mu-law or learned, and the
 * serving default clamps the log-mel value at -1.5 where the released config says -7.0). With L
 * clamped to [min_value, max_value] and u = (L - min_value) / (max_value - min_value):
 *   DMEL_QUANT_FLOOR  c = min(15, floor(16 u))                      (dmel_codes: [-7, 2])
 *   DMEL_QUANT_ROUND  c = floor(15 u + 1/2): the nearest of 16 reconstruction points
 *                     min_value + k (max_value - min_value) / 15, ties upward
 *   DMEL_QUANT_MULAW  c = min(15, floor(16 ln(1 + mu u) / ln(1 + mu)))
 * Arithmetic in fp32 like dmel_codes; codes agree with an fp64 evaluation except where the exact
 * log-mel value lies within 1e-4 of one of the mapping's 15 inner boundaries. */
typedef enum { DMEL_QUANT_FLOOR = 0, DMEL_QUANT_ROUND = 1, DMEL_QUANT_MULAW = 2 } dmel_quant_mode;

typedef struct {
  float min_value; /* clamp bottom (the released config: -7.0; the serving default: -1.5) */
  float max_value; /* clamp top (2.0); finite, > min_value */
  int mode;        /* dmel_quant_mode */
  float mu;        /* mu-law parameter (> 0, e.g. 255), ignored by the other modes */
} dmel_quantizer;

/* dmel_codes with the level mapping q (NULL: the default, exactly dmel_codes). Returns
 * DMEL_ERR_INVALID_ARG for a non-finite or empty clamp range, an unknown mode or mu <= 0 in
 * mu-law mode. Codes from here feed dmel_embed / dmel_embed_rows unchanged. */
dmel_status dmel_codes_q(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets, int n_clips,
                         int64_t n_frames, const float *tails, float *tails_out, uint8_t *codes,
                         const dmel_quantizer *q, dmel_stream_t stream);

/* ---- Sentinel expansion and splice ("Inside Inkling: Audio Design", Part 3 · Inference: at
 * serve time one audio item is a single sentinel token that expands into f d-mel frame
 * positions, and the server reports the realised count as audio_tokens).
 *
 * dmel_splice_plan (host, pure): a token sequence of seq_len positions holds n_items audio
 * sentinels at the strictly increasing positions h_sentinel_pos[0 .. n_items); item i is clip i,
 * whose frames are [h_frame_offsets[i], h_frame_offsets[i + 1]) (from dmel_frame_offsets). Each
 * sentinel is replaced by its f_i frames in place, so the expanded sequence has
 * seq_len + sum_i (f_i - 1) positions (a clip with no frame leaves no position). Outputs (each
 * may be NULL):
 *   h_token_pos    [seq_len]: the expanded position of each original position, -1 for sentinels
 *   h_frame_rows   [h_frame_offsets[n_items]]: the expanded position of each frame, in frame order
 *                  (the out_rows of dmel_embed_rows / dmel_forward_rows)
 *   h_expanded_len the expanded sequence length
 *   h_audio_tokens sum_i f_i, the count the server reports
 * Returns DMEL_ERR_INVALID_ARG (writing nothing) when seq_len < 0, n_items < 0, a sentinel
 * position is outside [0, seq_len) or not strictly increasing, or the frame offsets do not start
 * at 0 and increase. */
dmel_status dmel_splice_plan(const int64_t *h_sentinel_pos, int n_items, const int64_t *h_frame_offsets,
                             int64_t seq_len, int64_t *h_token_pos, int64_t *h_frame_rows,
                             int64_t *h_expanded_len, int64_t *h_audio_tokens);

/* dmel_embed and dmel_forward writing frame f's vector to row out_rows[f] of out instead of row f:
 * out is the decoder's input sequence [out_n_rows x embed_dim] (out_dtype), out_rows a device
 * int64 [n_frames] array (usually dmel_splice_plan's h_frame_rows, copied to the device). Rows
 * that no frame maps to are left as they are (the text tokens' embeddings). A row index outside
 * [0, out_n_rows) is not written and sets DMEL_DEVERR_OUT_ROW; rows mapped twice end up holding
 * one of the two frames. Every other argument, the workspace included, is as in dmel_embed /
 * dmel_forward. */
dmel_status dmel_embed_rows(const uint8_t *codes, int64_t n_frames, const void *table, dmel_dtype table_dtype,
                            int embed_dim, const void *rms_weight, float eps, void *out, const int64_t *out_rows,
                            int64_t out_n_rows, dmel_dtype out_dtype, void *workspace, size_t workspace_bytes,
                            dmel_stream_t stream);
dmel_status dmel_forward_rows(const float *wav, const int64_t *sample_offsets, const int64_t *frame_offsets,
                              int n_clips, int64_t n_frames, const float *tails, float *tails_out, const void *table,
                              dmel_dtype table_dtype, int embed_dim, const void *rms_weight, float eps, void *out,
                              const int64_t *out_rows, int64_t out_n_rows, dmel_dtype out_dtype, uint8_t *codes_out,
                              void *workspace, size_t workspace_bytes, dmel_stream_t stream);

/* ---- ShortConv ("Inside Inkling: Audio Design", Part 3 · Inference: the decoder's per-channel
 * causal convolutions of width W = 4, applied after the key/value projections and on the
 * residual-branch outputs, with a small per-request convolution state):
 *     y[t, c] = x[t, c] + sum_{d=0}^{3} weights[c * 4 + d] * x[t - d, c]
 * within each sequence s of tokens [seq_offsets[s], seq_offsets[s + 1]).
 * x            [n_tokens x channels] in dtype (fp32 or bf16), device, 16-byte aligned
 * seq_offsets  device int64 [n_seq + 1], 0 = seq_offsets[0] <= ... <= seq_offsets[n_seq] = n_tokens
 * channels     a positive multiple of 8
 * weights      device fp32 [channels x 4], 16-byte aligned
 * state        NULL (new requests: zeros before each sequence) or device [n_seq x 3 x channels] in
 *              dtype: row 3 + j holds x[j] for j = -3, -2, -1 of sequence s
 * state_out    NULL or [n_seq x 3 x channels]: the last three inputs each sequence ends with
 *              (taken from the state where a sequence is shorter than three); may be state
 * y            [n_tokens x channels] in dtype; must not overlap x or state
 * Sums in fp32, y rounded to dtype (bf16: nearest even). Offsets that do not describe the token
 * range read as zero inputs and set DMEL_DEVERR_OFFSETS. Asynchronous on stream. */
dmel_status dmel_shortconv(const void *x, const int64_t *seq_offsets, int n_seq, int64_t n_tokens, int channels,
                           const float *weights, const void *state, void *state_out, void *y, dmel_dtype dtype,
                           dmel_stream_t stream);

/* ---- hMLP patchifier (vision; "Inside Inkling: Audio Design", Part 1 · Modeling: a 4-layer
 * hMLP over 40x40 patches; "Why Thinking Machines Built Inkling Without a Vision Encoder":
 * linear layers progressively merge pixels into one embedding per patch). The pages give no
 * widths: the caller chooses them. Stage 1 maps every 5x5 pixel block of a patch (75 values in
 * row, column, channel order) to d1 features; stages 2, 3, 4 map every 2x2 group of the previous
 * stage's grid (the four vectors concatenated top-left, top-right, bottom-left, bottom-right) to
 * d2, d3 and dim features. Bias, LayerNorm (eps 1e-6, gain, shift) and GELU (u Phi(u), with
 * erfc from Abramowitz & Stegun 7.1.26: absolute error at most 1.5e-7) follow stages 1-3, bias
 * alone stage 4; every stage's output is stored in bf16, products sum in fp32. */
typedef struct {
  int d1, d2, d3, dim;            /* stage widths, each a positive multiple of 8 */
  const void *w1, *w2, *w3, *w4;  /* bf16 row-major [75 x d1], [4 d1 x d2], [4 d2 x d3], [4 d3 x dim] */
  const float *b1, *b2, *b3, *b4; /* fp32 biases [d1], [d2], [d3], [dim] */
  const float *g1, *g2, *g3;      /* fp32 LayerNorm gains [d1], [d2], [d3] */
  const float *be1, *be2, *be3;   /* fp32 LayerNorm shifts */
} dmel_hmlp_weights;              /* all device pointers, 16-byte aligned */

/* Bytes of device workspace dmel_hmlp needs for n_patches patches (0 when none). */
size_t dmel_hmlp_workspace_size(int64_t n_patches, const dmel_hmlp_weights *w);

/* images   bf16 [n_images x height x width x 3] (channel last), device, 16-byte aligned;
 *          height and width multiples of 40
 * out      bf16 [n_images * (height / 40) * (width / 40) x dim], patches in raster order
 * Stage 1 (d1 a multiple of 256, at most 1536; fewer than 2^31 pixel blocks) runs in one
 * tensor-core kernel of the library;
 * otherwise, and for stages 2-4, the products run on the library's tensor-core GEMM (bf16 x bf16,
 * fp32 sums, 256 x 192 tiles on CTA pairs) with the bias, LayerNorm and GELU in the library's row
 * kernel. Asynchronous on stream. */
dmel_status dmel_hmlp(const void *images, int n_images, int height, int width, const dmel_hmlp_weights *w, void *out,
                      void *workspace, size_t workspace_bytes, dmel_stream_t stream);

/* Reads (and, when clear != 0, clears) the device error word of the current device. This call
 * synchronises the device. *h_bits receives DMEL_DEVERR_* bits (0 = no error). */
dmel_status dmel_get_device_error(uint32_t *h_bits, int clear);

/* Human-readable name of a status code (static string, never NULL). */
const char *dmel_status_string(dmel_status status);

/* Number of kernel launches the last successful call on this host thread issued (for launch
 * accounting in benchmarks; 0 after a call that launched nothing). */
int dmel_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* DMEL_H */
