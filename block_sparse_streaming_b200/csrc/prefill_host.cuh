// prefill_host.cuh - host-side pipeline of loza_ssa_prefill_host: the prefill of
// a packed batch of sequences whose tensors live in host memory, streamed
// through the GPU in chunks of query blocks (each chunk inside one sequence)
// so that the PCIe copies in both directions overlap each other and the
// kernels.
//
// A query in block j reads the sink blocks 0 .. s-1 and the local blocks
// j-l+1 .. j (LongCat ZigZag Attention, page 1 section 01 (1)-(2)). A chunk of
// own query blocks [j0, j1) therefore needs the K/V rows of the sinks, of the
// halo blocks j0-l+1 .. j0-1 and of its own blocks. It runs the one-GPU prefill
// on the local sequence [sinks | halo | own]: local block t = j - j0 + s + l - 1
// of own block j has the window {0 .. s-1} U {t-l+1 .. t}, which is exactly
// the sinks, the halo and the own blocks up to j, so the own rows come out as
// in the whole-sequence prefill (the same kernel, the same keys in the same
// order). The prepended query rows are zeros; their outputs are not copied
// back. A chunk with j0 <= s + l - 1 has no gap between sinks and halo: its
// local sequence is simply rows [0, end of chunk), with j0 prepended blocks.
// The unbounded (full causal) window runs as one chunk.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <vector>

namespace loza {
namespace {

constexpr int kHostSlots = 3;          // chunks in flight: copy in, compute, copy out
constexpr int64_t kHostChunks = 16;    // aim: about this many chunks per sequence
constexpr int64_t kHostMinBlocks = 8;  // chunk size bounds, in blocks of 128 rows
constexpr int64_t kHostMaxBlocks = 64;

struct HostChunkPlan {
  int64_t nb;        // blocks in the sequence
  int64_t cb;        // own blocks per chunk
  int64_t n_chunks;
  int64_t pre_max;   // prepended blocks at most
  int64_t rows_max;  // local rows of the largest chunk
};

HostChunkPlan host_chunk_plan(int64_t seq_len, const loza_ssa_params& p) {
  HostChunkPlan h;
  h.nb = (seq_len + kTile - 1) / kTile;
  if (p.n_local == LOZA_UNBOUNDED) {
    h.pre_max = 0;
    h.cb = h.nb;
  } else {
    h.pre_max = (int64_t)p.n_sink + p.n_local - 1;
    int64_t cb = (h.nb + kHostChunks - 1) / kHostChunks;
    // at least as many own blocks as prepended ones, so that the zero query
    // rows cost at most as much as the own rows
    cb = std::max(cb, std::max(h.pre_max, kHostMinBlocks));
    cb = std::min(cb, std::max(kHostMaxBlocks, h.pre_max));
    h.cb = std::min(cb, h.nb);
  }
  h.n_chunks = (h.nb + h.cb - 1) / h.cb;
  // a local sequence never holds more rows than the prefix up to its chunk's end
  h.rows_max = std::min((h.pre_max + h.cb) * kTile, seq_len);
  return h;
}

// One chunk: own query rows [q0, q1), `pre` prepended blocks, and the K/V rows
// copied into the local sequence as up to two runs of host rows.
struct HostChunk {
  int64_t q0, q1, pre;
  int64_t src0, n0, src1, n1;  // run 0 -> local row 0, run 1 -> local row n0
  int64_t local_len() const { return pre * kTile + (q1 - q0); }
};

HostChunk host_chunk(const HostChunkPlan& h, int64_t c, int64_t seq_len, const loza_ssa_params& p) {
  HostChunk k;
  const int64_t j0 = c * h.cb;
  const int64_t j1 = std::min(j0 + h.cb, h.nb);
  k.q0 = j0 * kTile;
  k.q1 = std::min(j1 * kTile, seq_len);
  if (p.n_local == LOZA_UNBOUNDED || j0 <= h.pre_max) {
    k.pre = j0;
    k.src0 = 0;
    k.n0 = k.q1;
    k.src1 = 0;
    k.n1 = 0;
  } else {
    k.pre = h.pre_max;
    k.src0 = 0;
    k.n0 = (int64_t)p.n_sink * kTile;
    k.src1 = (j0 - p.n_local + 1) * kTile;
    k.n1 = k.q1 - k.src1;
  }
  return k;
}

// Upper bound of the chunks of a packed batch: a sequence of nb blocks is one
// chunk if nb < kHostMinBlocks, otherwise chunks of at least kHostMinBlocks
// blocks, at most nb / kHostMinBlocks + 1 of them.
int64_t host_chunk_cap(int32_t batch, int64_t total_tokens) {
  return 2 * (int64_t)batch + total_tokens / (kTile * kHostMinBlocks) + 1;
}

struct HostLayout {
  size_t cu_off, pf_off, pf_bytes, slot_off, slot_bytes;
  size_t q_off, k_off, v_off, o_off, l_off;  // within a slot
  int slots;
  size_t total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace of a packed batch: slots sized for the longest sequence's largest
// chunk (chunks grow with the sequence), the local cu_seqlens of every chunk.
HostLayout host_layout(const HostChunkPlan& h, int64_t chunk_cap, size_t pf_bytes, int32_t n_heads,
                       int32_t n_kv_heads, int32_t d_qk, int32_t d_v) {
  HostLayout w;
  const size_t rows = (size_t)h.rows_max;
  w.slots = (int)std::min<int64_t>(kHostSlots, chunk_cap);
  w.cu_off = 0;
  w.pf_off = align256((size_t)chunk_cap * 2 * sizeof(int32_t));
  w.pf_bytes = pf_bytes;
  w.slot_off = align256(w.pf_off + pf_bytes);
  w.q_off = 0;
  w.k_off = align256(w.q_off + rows * n_heads * d_qk * 2);
  w.v_off = align256(w.k_off + rows * n_kv_heads * d_qk * 2);
  w.o_off = align256(w.v_off + rows * n_kv_heads * d_v * 2);
  w.l_off = align256(w.o_off + rows * n_heads * d_v * 2);
  w.slot_bytes = align256(w.l_off + rows * n_heads * sizeof(float));
  w.total = w.slot_off + (size_t)w.slots * w.slot_bytes;
  return w;
}

bool host_shape_ok(int32_t n_heads, int32_t n_kv_heads, int32_t d_qk, int32_t d_v) {
  if (n_heads < 1 || n_kv_heads < 1 || n_heads % n_kv_heads != 0) return false;
  if (!(n_kv_heads == 1 || n_kv_heads == n_heads)) return false;
  return (d_qk == 64 && d_v == 64) || (d_qk == 192 && d_v == 128) ||
         (d_qk == 576 && d_v == 512 && n_kv_heads == 1 && n_heads % 2 == 0);
}

// Two non-blocking copy streams and the events that order them against the
// caller's stream, created on first use per device and kept until exit.
struct HostPipe {
  std::mutex mu;
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t in_done[kHostSlots] = {}, run_done[kHostSlots] = {}, out_done[kHostSlots] = {};
};
HostPipe g_host_pipes[kMaxDevices];

void host_pipe_release(HostPipe& hp) {
  if (hp.h2d) cudaStreamDestroy(hp.h2d);
  if (hp.d2h) cudaStreamDestroy(hp.d2h);
  if (hp.start) cudaEventDestroy(hp.start);
  for (int i = 0; i < kHostSlots; ++i) {
    if (hp.in_done[i]) cudaEventDestroy(hp.in_done[i]);
    if (hp.run_done[i]) cudaEventDestroy(hp.run_done[i]);
    if (hp.out_done[i]) cudaEventDestroy(hp.out_done[i]);
    hp.in_done[i] = hp.run_done[i] = hp.out_done[i] = nullptr;
  }
  hp.h2d = hp.d2h = nullptr;
  hp.start = nullptr;
}

// All or nothing: a failed creation releases what was created before it.
bool host_pipe_init(HostPipe& hp) {
  if (hp.ready) return true;
  bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; ok && i < kHostSlots; ++i)
    ok = cudaEventCreateWithFlags(&hp.in_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.run_done[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp.out_done[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    host_pipe_release(hp);
    return false;
  }
  hp.ready = true;
  return true;
}

}  // namespace
}  // namespace loza
