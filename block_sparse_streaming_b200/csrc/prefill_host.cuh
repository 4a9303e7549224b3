// prefill_host.cuh - host-side pipeline of loza_ssa_prefill_host: the prefill of
// a packed batch of sequences whose tensors live in host memory, streamed
// through the GPU in chunks of query blocks (each chunk inside one sequence)
// so that the PCIe copies in both directions overlap each other and the
// kernels.
//
// The window of query i (LongCat ZigZag Attention, page 1 section 01 (1)-(2),
// blocks of b tokens) is the sink rows [0, s*b) and the local rows [lo(i), i],
// lo(i) = max(0, (floor(i/b) - l + 1) * b). A chunk of own query rows [q0, q1)
// (q0 a multiple of U = max(b, 128)) therefore needs the K/V rows of the sinks,
// of the halo [q0 - (l-1)*b, q0) and its own rows. It runs the one-GPU prefill
// on the local sequence [sinks | gap | halo | own], whose prefix (sinks, gap of
// zero rows, halo) holds P rows: the smallest multiple of U that fits the sinks
// rounded up to whole 128-row tiles, plus the halo (P = (s + l - 1) * 128 and
// no gap for b = 128). An own row i sits at local row i - q0 + P; q0 and P are
// multiples of U, so floor(i/b) moves by whole blocks and the local window is
// the sinks plus the halo and own rows up to i, the keys of the whole sequence;
// the gap lies past the sinks and before every own row's window. Every row and
// key keeps its place in its 128-row tile and the halo never shares a tile with
// the sinks, so the kernels walk the same tiles in the same order and the own
// rows come out bit for bit as in the whole-sequence prefill. The prepended
// query rows are zeros; their outputs are not copied back. A chunk with q0 <= P
// runs on rows [0, q1) of the sequence itself (q0 rows prepended). The
// unbounded (full causal) window runs as one chunk.
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
constexpr int64_t kHostMinRows = 1024; // chunk size bounds, in rows (rounded to whole units)
constexpr int64_t kHostMaxRows = 8192;

struct HostChunkPlan {
  int64_t unit;      // rows per unit: max(b, 128)
  int64_t nu;        // units in the sequence
  int64_t cu;        // own units per chunk
  int64_t n_chunks;
  int64_t pre;       // rows of the prefix [sinks | gap | halo] of a chunk past it (0: unbounded)
  int64_t rows_max;  // local rows of the largest chunk
};

HostChunkPlan host_chunk_plan(int64_t seq_len, const loza_ssa_params& p) {
  HostChunkPlan h;
  const int64_t b = p.block_size;
  h.unit = std::max<int64_t>(b, kTile);
  h.nu = (seq_len + h.unit - 1) / h.unit;
  if (p.n_local == LOZA_UNBOUNDED) {
    h.pre = 0;
    h.cu = h.nu;
  } else {
    const int64_t sink_tiles_rows = ((int64_t)p.n_sink * b + kTile - 1) / kTile * kTile;
    const int64_t halo = ((int64_t)p.n_local - 1) * b;
    h.pre = (sink_tiles_rows + halo + h.unit - 1) / h.unit * h.unit;
    const int64_t pre_units = h.pre / h.unit;
    const int64_t min_units = (kHostMinRows + h.unit - 1) / h.unit;
    const int64_t max_units = std::max<int64_t>(1, kHostMaxRows / h.unit);
    int64_t cu = (h.nu + kHostChunks - 1) / kHostChunks;
    // at least as many own rows as prepended ones, so that the zero query
    // rows cost at most as much as the own rows
    cu = std::max(cu, std::max(pre_units, min_units));
    cu = std::min(cu, std::max(max_units, pre_units));
    h.cu = std::min(cu, h.nu);
  }
  h.n_chunks = (h.nu + h.cu - 1) / h.cu;
  // a local sequence never holds more rows than the prefix up to its chunk's end
  h.rows_max = std::min(h.pre + h.cu * h.unit, seq_len);
  return h;
}

// One chunk: own query rows [q0, q1), `pre` prepended rows, and the K/V rows
// of the local sequence: run 0 of host rows -> local row 0, then `gap` zero
// rows, then run 1 -> local row n0 + gap.
struct HostChunk {
  int64_t q0, q1, pre;
  int64_t src0, n0, gap, src1, n1;
  int64_t local_len() const { return pre + (q1 - q0); }
};

HostChunk host_chunk(const HostChunkPlan& h, int64_t c, int64_t seq_len, const loza_ssa_params& p) {
  HostChunk k;
  k.q0 = c * h.cu * h.unit;
  k.q1 = std::min(k.q0 + h.cu * h.unit, seq_len);
  if (p.n_local == LOZA_UNBOUNDED || k.q0 <= h.pre) {
    k.pre = k.q0;
    k.src0 = 0;
    k.n0 = k.q1;
    k.gap = 0;
    k.src1 = 0;
    k.n1 = 0;
  } else {
    const int64_t b = p.block_size;
    k.pre = h.pre;
    k.src0 = 0;
    k.n0 = (int64_t)p.n_sink * b;
    k.src1 = k.q0 - ((int64_t)p.n_local - 1) * b;
    k.gap = h.pre - k.n0 - (k.q0 - k.src1);
    k.n1 = k.q1 - k.src1;
  }
  return k;
}

// Upper bound of the chunks of a packed batch: every chunk of a sequence but
// its last holds at least kHostMinRows own rows, so a sequence of L rows has at
// most L / kHostMinRows + 1 chunks.
int64_t host_chunk_cap(int32_t batch, int64_t total_tokens) {
  return 2 * (int64_t)batch + total_tokens / kHostMinRows + 1;
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
