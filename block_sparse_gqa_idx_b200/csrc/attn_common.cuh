// attn_common.cuh -- what the KV-outer kernels share: the query-chunk
// workspace, the inverse index's parameters and launcher, and small device
// helpers (inverse index in inv_index.cu; its users: the forward in
// sparse_attn.cu, the KL-loss fusion in index_lse.cu, the backward in
// sparse_bwd.cu).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"

namespace msa {

// Largest per-CTA key histogram of the inverse index (H_kv * B keys).
constexpr size_t kMaxHistBytes = 192 * 1024;
constexpr int kRowsPerTile = 128;
// Queries per chunk: bounds the partial-output workspace.  Chunks are kept
// large so that every (group, block) list holds many queries per chunk: K/V
// blocks are then reused over long runs of tiles (small chunks would keep the
// gathered Q in L2 but re-read K/V for nearly every tile at 1M tokens).
constexpr int kMaxChunk = 1 << 17;
// Queries per window of the inverse index's keys.  One window per chunk:
// keys are (group, block) and a key's list spans the whole chunk, so a K/V
// block is reused over long runs of tiles.  (Windows of 8192 queries, which
// keep a window's gathered Q rows in L2, were measured slower: a key's list
// per window is then only a few tiles long -- one at 1M tokens -- and the
// K/V reloads cost more than the Q reuse saves.)
constexpr int kWindow = kMaxChunk;

// Rows per query inside an MMA tile: the group's G heads, or 8 heads (one
// 128-byte swizzle atom) when G < 8 (the extra heads are computed and dropped).
inline int rows_per_query(int G) { return G >= 8 ? G : 8; }

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct ChunkBufs {
  int32_t* counts;    // [nkeys]
  int32_t* offsets;   // [nkeys + 1]
  int32_t* tile_off;  // [nkeys + 1]
  int32_t* cursor;    // [nkeys]
  int32_t* n_tiles;   // [4]
  int32_t* block_sums;  // [2 * scan blocks]: per block of keys, (count, tiles), then their offsets
  int4* tile_meta;       // [tiles]: per tile (key, first entry, queries, the key's end tile)
  uint32_t* entries;  // [Nc * H_kv * k]
  __half* part_o;     // [Nc * H_kv * k, d_h / 8, G, 8]: per slot, 16-byte d-chunks head-minor
  float* part_lse;    // [Nc * H_kv * k, G]
};

inline ChunkBufs carve(void* ws, int64_t Nc, int H_q, int H_kv, int d_h, int kk, int64_t nkeys,
                size_t* total) {
  ChunkBufs c;
  uint8_t* p = static_cast<uint8_t*>(ws);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const int G = H_q / H_kv;
  const int64_t slots = Nc * H_kv * kk;
  c.part_o = reinterpret_cast<__half*>(take(sizeof(__half) * slots * G * d_h));
  c.part_lse = reinterpret_cast<float*>(take(sizeof(float) * slots * G));
  c.entries = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * slots));
  c.counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nkeys));
  c.cursor = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nkeys));
  c.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (nkeys + 1)));
  c.tile_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (nkeys + 1)));
  c.n_tiles = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * 4));
  c.block_sums = reinterpret_cast<int32_t*>(
      take(sizeof(int32_t) * 2 * ((nkeys + 4095) / 4096 + 1)));
  // tiles <= entries / (smallest tile of 4 queries) + keys
  c.tile_meta = reinterpret_cast<int4*>(take(sizeof(int4) * (slots / 4 + nkeys + 1)));
  *total = off;
  return c;
}

inline int64_t chunk_len(int64_t N, int B_k) {
  int64_t c = N < kMaxChunk ? N : kMaxChunk;
  return (c + B_k - 1) / B_k * B_k;
}

// ------------------------------------------------------------------ step 1 --
// Keys of the inverse index: (query window w, group r, block b), key =
// (w * H_kv + r) * B + b, windows of Cw consecutive queries of the chunk.  The
// lists of one window are contiguous in key order, so a schedule that walks
// the tiles in key order works through one window of queries at a time and
// their gathered Q rows stay in L2.
struct InvParams {
  const int32_t* idx;
  int64_t q0, nq;  // chunk [q0, q0 + nq)
  int H_kv, B_k, kk;
  int64_t B;  // blocks (all sequences' blocks, numbered globally, when qinfo is set)
  // packed sequences: per token {first token, first global block} of its
  // sequence; null for one sequence
  const int2* qinfo;
  int Tq;
  int Cw, W;  // queries per window, windows in the chunk
  ChunkBufs c;
  DevStatus* status;
};

constexpr int kScanThreads = 1024;
constexpr int kScanPerThread = 4;
constexpr int kScanBlockKeys = kScanThreads * kScanPerThread;
static_assert(kScanBlockKeys == 4096, "the workspace carve sizes the block sums for 4096 keys");

inline int64_t inv_nkeys(int64_t nq, int Cw, int H_kv, int64_t B) {
  return (nq + Cw - 1) / Cw * H_kv * B;
}
inline int64_t scan_blocks(int64_t nkeys) { return (nkeys + kScanBlockKeys - 1) / kScanBlockKeys; }

// Query i's sequence: its first token and the global number of its block 0
// ({0, 0} for one sequence).
__device__ __forceinline__ int2 seq_of(const int2* qinfo, int64_t i) {
  return qinfo != nullptr ? qinfo[i] : make_int2(0, 0);
}

// The key whose tile range holds tile t (tile_off[key] <= t < tile_off[key+1]).
__device__ __forceinline__ int find_key(const int32_t* tile_off, int64_t nkeys, int t) {
  int64_t lo = 0, hi = nkeys;  // tile_off[lo] <= t < tile_off[hi]
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (tile_off[mid] <= t) lo = mid;
    else hi = mid;
  }
  return static_cast<int>(lo);
}

// The query chunk's inverse index: count, scan (tile offsets and per-tile
// records), scatter.  inv_setup sizes the histogram kernels for nlocal keys.
cudaError_t inv_setup(int64_t nlocal, int sms, size_t* hist_bytes, int* hist_ctas);
void launch_inv_index(const InvParams& ip, size_t hist_bytes, int hist_ctas, int sms,
                      cudaStream_t stream);

}  // namespace msa
