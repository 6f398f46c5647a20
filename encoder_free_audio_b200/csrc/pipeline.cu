// dmel_forward_host: waveforms in host memory to frame vectors in host memory, with the
// host-to-device copies, the kernels and the device-to-host copies overlapped chunk by chunk.
//
// The batch's frames are cut into chunks of at most chunk_frames frames (a cut may fall inside a
// clip). A chunk is a list of pieces, one per clip it touches: frames [t0, t1) of clip c need
// the clip's samples [800 (t0 - 1), 800 t1) under the causal framing ("Inside Inkling: Audio
// Design", Part 1 · Modeling: hop 800, window 1600), so a piece that starts inside its clip
// carries the 800 samples before it as its tail, exactly like a streaming call.
//
// Two device buffer sets alternate; per chunk i (buffer set b = i mod 2):
//   copy-in stream   waits until the kernels of chunk i - 2 have read set b, copies the chunk's
//                    samples (one contiguous range of the host batch) and its first piece's tail;
//   caller's stream  waits for the copy-in and for the copy-out of chunk i - 2 (set b's vectors),
//                    runs the codes and embedding kernels of the chunk;
//   copy-out stream  waits for those kernels and copies the chunk's vectors (and codes) to host.
// The caller's stream finally waits for the last copy-out, so work queued after the call on that
// stream (or a synchronisation of it) sees every result in host memory.
#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace dmel {
namespace {

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

struct Piece {
  int clip;
  int64_t t0, t1;  // frames of the clip in this chunk
};

struct Chunk {
  int64_t f0, f1;      // frames of the batch
  int p0, p1;          // pieces [p0, p1) of the plan
  int64_t s_lo, s_hi;  // host samples copied: [s_lo, s_hi) (s_lo includes the tail when there is one)
  bool tail;           // the first piece starts inside its clip
  int64_t table_off;   // offset (in int64) of this chunk's piece offsets in the offsets table
};

struct Plan {
  int64_t n_frames = 0;
  std::vector<Piece> pieces;
  std::vector<Chunk> chunks;
  std::vector<int64_t> table;  // per chunk: sample offsets [n + 1], then frame offsets [n + 1]
  int max_pieces = 0;
  int64_t max_samples = 0;     // largest s_hi - s_lo
  int64_t chunk_frames = 0;
};

// Cuts the batch into chunks. h_sample_offsets must be valid (checked by the caller).
void make_plan(const int64_t *so, int n_clips, int64_t chunk_frames, Plan *P) {
  std::vector<int64_t> fo(n_clips + 1);
  fo[0] = 0;
  for (int c = 0; c < n_clips; ++c) fo[c + 1] = fo[c] + (so[c + 1] - so[c]) / kHop;
  P->n_frames = fo[n_clips];
  P->chunk_frames = chunk_frames;
  int c = 0;
  for (int64_t f0 = 0; f0 < P->n_frames; f0 += chunk_frames) {
    const int64_t f1 = std::min(P->n_frames, f0 + chunk_frames);
    while (fo[c + 1] <= f0) ++c;  // first clip with a frame at or after f0 (skips clips with none)
    Chunk ch;
    ch.f0 = f0;
    ch.f1 = f1;
    ch.p0 = (int)P->pieces.size();
    for (int k = c; k < n_clips && fo[k] < f1; ++k) {
      if (fo[k + 1] == fo[k]) continue;  // no frame
      P->pieces.push_back(Piece{k, std::max(f0, fo[k]) - fo[k], std::min(f1, fo[k + 1]) - fo[k]});
    }
    ch.p1 = (int)P->pieces.size();
    const Piece &first = P->pieces[ch.p0], &last = P->pieces[ch.p1 - 1];
    ch.tail = first.t0 > 0;
    const int64_t start0 = so[first.clip] + (int64_t)kHop * first.t0;
    ch.s_lo = start0 - (ch.tail ? kHop : 0);
    ch.s_hi = so[last.clip] + (int64_t)kHop * last.t1;
    // piece p spans [start_p, start_{p+1}) of the copied samples (the last: up to s_hi); a span
    // may run past the piece's last frame (a clip's unused remainder, clips with no frame), which
    // the codes kernel never reads: its frames come from the frame offsets
    ch.table_off = (int64_t)P->table.size();
    const int n = ch.p1 - ch.p0;
    for (int p = ch.p0; p < ch.p1; ++p)
      P->table.push_back(so[P->pieces[p].clip] + (int64_t)kHop * P->pieces[p].t0 - start0);
    P->table.push_back(ch.s_hi - start0);
    int64_t acc = 0;
    P->table.push_back(0);
    for (int p = ch.p0; p < ch.p1; ++p) {
      acc += P->pieces[p].t1 - P->pieces[p].t0;
      P->table.push_back(acc);
    }
    P->max_pieces = std::max(P->max_pieces, n);
    P->max_samples = std::max(P->max_samples, ch.s_hi - ch.s_lo);
    P->chunks.push_back(ch);
  }
}

// Workspace layout: offsets table, then per buffer set: samples [max_samples] (the first
// piece's first sample at float 0), tails [max_pieces x 800], codes [chunk_frames x 80],
// vectors [chunk_frames x D]; then the embedding's scratch.
struct Layout {
  size_t table, wav[2], tails[2], codes[2], out[2], embed, total;
};

Layout layout(const Plan &P, int D, size_t out_es, dmel_dtype table_dtype, int with_rms) {
  Layout L;
  size_t off = 0;
  L.table = off;
  off += round256(P.table.size() * sizeof(int64_t));
  const int64_t cf = std::min(P.chunk_frames, P.n_frames);
  for (int b = 0; b < 2; ++b) {
    L.wav[b] = off;
    off += round256((size_t)P.max_samples * sizeof(float));
    L.tails[b] = off;
    off += round256((size_t)P.max_pieces * kHop * sizeof(float));
    L.codes[b] = off;
    off += round256((size_t)cf * kMel);
    L.out[b] = off;
    off += round256((size_t)cf * (size_t)D * out_es);
  }
  L.embed = off;
  off += round256(embed_workspace_bytes(cf, D, table_dtype, with_rms));
  L.total = off;
  return L;
}

struct Streams {
  cudaStream_t in = nullptr, out = nullptr;
};
std::mutex g_streams_mu;
Streams g_streams[256];

// The copy streams of the current device, created once (non-blocking).
cudaError_t copy_streams(Streams *s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 256) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_streams_mu);
  Streams &st = g_streams[dev];
  if (!st.in) {
    if ((e = cudaStreamCreateWithFlags(&st.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&st.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
  }
  *s = st;
  return cudaSuccess;
}

}  // namespace

size_t forward_host_workspace_bytes(const int64_t *h_so, int n_clips, int D, dmel_dtype table_dtype,
                                    dmel_dtype out_dtype, int with_rms, int64_t chunk_frames) {
  Plan P;
  make_plan(h_so, n_clips, chunk_frames, &P);
  if (P.n_frames == 0) return 0;
  return layout(P, D, out_dtype == DMEL_BF16 ? 2 : 4, table_dtype, with_rms).total;
}

int64_t debug_forward_host_plan(const int64_t *h_so, int n_clips, int64_t chunk_frames, int64_t *h_plan,
                                int64_t cap) {
  Plan P;
  make_plan(h_so, n_clips, chunk_frames, &P);
  int64_t len = 0;
  auto put = [&](int64_t v) {
    if (len < cap) h_plan[len] = v;
    ++len;
  };
  for (const Chunk &ch : P.chunks) {
    const int n = ch.p1 - ch.p0;
    put(ch.f0);
    put(ch.f1);
    put(ch.s_lo);
    put(ch.s_hi);
    put(ch.tail ? 1 : 0);
    put(n);
    for (int i = 0; i < 2 * (n + 1); ++i) put(P.table[ch.table_off + i]);
  }
  return len;
}

cudaError_t run_forward_host(const float *h_wav, const int64_t *h_so, int n_clips, const void *table,
                             dmel_dtype table_dtype, int D, const void *rms_weight, float eps, void *h_out,
                             dmel_dtype out_dtype, uint8_t *h_codes, int64_t chunk_frames, void *workspace,
                             size_t workspace_bytes, uint32_t *err, int num_sms, cudaStream_t stream,
                             int *launches, bool *too_small) {
  Plan P;
  make_plan(h_so, n_clips, chunk_frames, &P);
  *too_small = false;
  if (P.n_frames == 0) return cudaSuccess;
  const size_t out_es = out_dtype == DMEL_BF16 ? 2 : 4;
  const Layout L = layout(P, D, out_es, table_dtype, rms_weight != nullptr);
  if (!workspace || workspace_bytes < L.total) {
    *too_small = true;
    return cudaSuccess;
  }
  Streams cs;
  cudaError_t e = copy_streams(&cs);
  if (e != cudaSuccess) return e;
  uint8_t *ws = static_cast<uint8_t *>(workspace);
  int64_t *d_table = reinterpret_cast<int64_t *>(ws + L.table);

  // events: start (caller's stream), and per buffer set: copied in, computed, copied out
  cudaEvent_t ev_start, ev_in[2], ev_comp[2], ev_out[2];
  cudaEvent_t *all[7] = {&ev_start, &ev_in[0], &ev_in[1], &ev_comp[0], &ev_comp[1], &ev_out[0], &ev_out[1]};
  int made = 0;
  for (; made < 7; ++made)
    if ((e = cudaEventCreateWithFlags(all[made], cudaEventDisableTiming)) != cudaSuccess) break;
  auto destroy = [&] {
    for (int i = 0; i < made; ++i) cudaEventDestroy(*all[i]);  // released once their work is done
  };
  if (e != cudaSuccess) {
    destroy();
    return e;
  }
  auto fail = [&](cudaError_t x) {
    destroy();
    return x;
  };
  // the copy streams start after the work already queued on the caller's stream (which may
  // still be producing the inputs or reading the outputs of an earlier call)
  if ((e = cudaEventRecord(ev_start, stream)) != cudaSuccess) return fail(e);
  if ((e = cudaStreamWaitEvent(cs.in, ev_start, 0)) != cudaSuccess) return fail(e);
  if ((e = cudaStreamWaitEvent(cs.out, ev_start, 0)) != cudaSuccess) return fail(e);
  // the piece offsets of every chunk (a small pageable copy, staged by the driver before it
  // returns), and the tails of both buffer sets zeroed once: only row 0 ever changes
  if ((e = cudaMemcpyAsync(d_table, P.table.data(), P.table.size() * sizeof(int64_t), cudaMemcpyHostToDevice,
                           cs.in)) != cudaSuccess)
    return fail(e);
  for (int b = 0; b < 2; ++b)
    if ((e = cudaMemsetAsync(ws + L.tails[b], 0, (size_t)P.max_pieces * kHop * sizeof(float), cs.in)) != cudaSuccess)
      return fail(e);

  for (size_t i = 0; i < P.chunks.size(); ++i) {
    const Chunk &ch = P.chunks[i];
    const int b = (int)(i & 1);
    float *d_wav = reinterpret_cast<float *>(ws + L.wav[b]);  // the first piece's first sample
    float *d_tails = reinterpret_cast<float *>(ws + L.tails[b]);
    uint8_t *d_codes = ws + L.codes[b];
    uint8_t *d_out = ws + L.out[b];
    const int n = ch.p1 - ch.p0;
    const int64_t nf = ch.f1 - ch.f0;
    // ---- copy in (set b is free once chunk i - 2's kernels are done)
    if (i >= 2 && (e = cudaStreamWaitEvent(cs.in, ev_comp[b], 0)) != cudaSuccess) return fail(e);
    const int64_t first = ch.s_lo + (ch.tail ? kHop : 0);
    if ((e = cudaMemcpyAsync(d_wav, h_wav + first, (size_t)(ch.s_hi - first) * sizeof(float), cudaMemcpyHostToDevice,
                             cs.in)) != cudaSuccess)
      return fail(e);
    if (ch.tail)
      e = cudaMemcpyAsync(d_tails, h_wav + ch.s_lo, kHop * sizeof(float), cudaMemcpyHostToDevice, cs.in);
    else if (i >= 2 && P.chunks[i - 2].tail)
      e = cudaMemsetAsync(d_tails, 0, kHop * sizeof(float), cs.in);
    if (e != cudaSuccess) return fail(e);
    if ((e = cudaEventRecord(ev_in[b], cs.in)) != cudaSuccess) return fail(e);
    // ---- kernels on the caller's stream (set b's vectors are free once copied out)
    if ((e = cudaStreamWaitEvent(stream, ev_in[b], 0)) != cudaSuccess) return fail(e);
    if (i >= 2 && (e = cudaStreamWaitEvent(stream, ev_out[b], 0)) != cudaSuccess) return fail(e);
    const int64_t *d_so = d_table + ch.table_off, *d_fo = d_so + n + 1;
    if ((e = launch_codes(d_wav, d_so, d_fo, n, nf, d_tails, nullptr, d_codes, err, num_sms, stream, launches)) !=
        cudaSuccess)
      return fail(e);
    if ((e = launch_embed(d_codes, nf, table, table_dtype, D, rms_weight, eps, d_out, out_dtype, ws + L.embed, err,
                          num_sms, stream, launches)) != cudaSuccess)
      return fail(e);
    if ((e = cudaEventRecord(ev_comp[b], stream)) != cudaSuccess) return fail(e);
    // ---- copy out
    if ((e = cudaStreamWaitEvent(cs.out, ev_comp[b], 0)) != cudaSuccess) return fail(e);
    if ((e = cudaMemcpyAsync(static_cast<uint8_t *>(h_out) + (size_t)ch.f0 * D * out_es, d_out,
                             (size_t)nf * D * out_es, cudaMemcpyDeviceToHost, cs.out)) != cudaSuccess)
      return fail(e);
    if (h_codes && (e = cudaMemcpyAsync(h_codes + (size_t)ch.f0 * kMel, d_codes, (size_t)nf * kMel,
                                        cudaMemcpyDeviceToHost, cs.out)) != cudaSuccess)
      return fail(e);
    if ((e = cudaEventRecord(ev_out[b], cs.out)) != cudaSuccess) return fail(e);
  }
  // the caller's stream ends after the last copy out
  const int last = (int)((P.chunks.size() - 1) & 1);
  if ((e = cudaStreamWaitEvent(stream, ev_out[last], 0)) != cudaSuccess) return fail(e);
  destroy();
  return cudaSuccess;
}

}  // namespace dmel
