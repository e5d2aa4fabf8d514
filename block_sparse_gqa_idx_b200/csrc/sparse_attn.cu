// sparse_attn.cu -- Main Branch (Eq. 8 with the causal rule of Eq. 1) as a
// KV-outer block-sparse attention on tcgen05, in three steps per query chunk:
//
//   1. inverse index: for every (group r, block b) the list of selection slots
//      (query i, slot s) that chose b -- count, exclusive scan (multi-CTA),
//      scatter, each CTA counting its range of slots in a shared-memory
//      histogram of the keys.  The scan also cuts each list into tiles of Tq
//      queries (Tq * rows-per-query = 128 MMA rows) and writes each tile's
//      (key, first entry, length), so hot blocks are split over many CTAs
//      with every output slot fixed in advance: no atomics on the outputs.
//   2. phase 1: one tile = one KV block (K_b, V_b by TMA) and the gathered
//      query rows that selected it (one TMA box per query: its group's heads).
//      S = Q K_b^T (UMMA, fp32 in TMEM) -> causal mask (only rows whose own
//      block is b) -> softmax by eight warps (two threads per row, exp2) ->
//      P / l (bf16) back into TMEM -> O = P V_b (UMMA with A in TMEM) -> O
//      written as an fp16 partial, with its natural-log LSE, into the row's
//      slot.
//   3. merge: per (query, head), LSE-weighted sum of its partials (split-K
//      softmax normalisation), bf16 output + fp32 LSE.
//
// The file also holds the KL-loss fusion's Index Branch normaliser LSE_idx
// (review "4.3 Sparse KL Loss Fusion"): the same inverse index in 16-slot
// tiles, each selected block's index-score LSE per slot (mma.sync), and a
// log-sum-exp over a row's slots.
//
// Source: xllm-io paper review, "核心公式" Eq. 8 and "4.2 Sparse Attention
// Kernel" (KV-outer with query gather, two-phase forward: partial outputs
// then a combine pass); chlience notes 5.4 (pre-scheduled tile chunking,
// slots assigned ahead, two-phase combine).
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <type_traits>

#include "msa_internal.h"

namespace msa {
namespace {

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

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

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

ChunkBufs carve(void* ws, int64_t Nc, int H_q, int H_kv, int d_h, int kk, int64_t nkeys,
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

int64_t chunk_len(int64_t N, int B_k) {
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

// The window-local key (r * B + global block) of entry e of the chunk, or -1
// when the entry selects nothing (-1 padding, or a block after the query's
// own).  Entry e is (query, group, slot) in the layout of I, so e is also the
// entry's output slot id and I is read contiguously.
__device__ __forceinline__ int inv_key(const InvParams& p, int64_t e, bool report_bad) {
  const int64_t per_q = static_cast<int64_t>(p.H_kv) * p.kk;
  const int64_t il = e / per_q;
  const int r = static_cast<int>((e - il * per_q) / p.kk);
  const int64_t i = p.q0 + il;
  const int32_t b = p.idx[p.q0 * per_q + e];
  if (b < -1 || b >= p.B) {
    if (report_bad) report(p.status, DEV_ERR_BAD_INDEX, 40, static_cast<int>(i), b);
    return -1;
  }
  const int2 sq = seq_of(p.qinfo, i);
  return (b >= 0 && b <= (i - sq.x) / p.B_k) ? r * static_cast<int>(p.B) + sq.y + b : -1;
}

// Inverse index with a per-CTA histogram of one window's keys in shared
// memory.  The grid is W x (CTAs per window); a CTA owns a contiguous range
// of its window's entries.  Counting: the CTA counts its entries per key in
// shared memory and adds each non-zero count to the global one with a single
// atomic.  Scattering: the CTA counts again, reserves each key's range of the
// key's list with one atomic on the key's cursor, and places every entry at a
// shared-memory atomic's position inside that range.
template <bool SCATTER>
__global__ void __launch_bounds__(512) inv_index_smem_kernel(const InvParams p) {
  extern __shared__ int32_t hist[];  // [H_kv * B]
  const int nlocal = static_cast<int>(p.H_kv * p.B);
  const int cpw = gridDim.x / p.W;
  const int w = blockIdx.x / cpw, cw = blockIdx.x - w * cpw;
  const int64_t per_q = static_cast<int64_t>(p.H_kv) * p.kk;
  const int64_t wq1 = min(static_cast<int64_t>(w + 1) * p.Cw, p.nq);
  const int64_t we0 = static_cast<int64_t>(w) * p.Cw * per_q, we1 = wq1 * per_q;
  const int64_t per = (we1 - we0 + cpw - 1) / cpw;
  const int64_t e0 = we0 + cw * per;
  const int64_t e1 = e0 + per < we1 ? e0 + per : we1;
  const int64_t kbase = static_cast<int64_t>(w) * nlocal;
  for (int j = threadIdx.x; j < nlocal; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int key = inv_key(p, e, !SCATTER);
    if (key >= 0) atomicAdd(&hist[key], 1);
  }
  __syncthreads();
  if constexpr (!SCATTER) {
    for (int j = threadIdx.x; j < nlocal; j += blockDim.x) {
      const int n = hist[j];
      if (n > 0) atomicAdd(&p.c.counts[kbase + j], n);
    }
  } else {
    for (int j = threadIdx.x; j < nlocal; j += blockDim.x) {
      const int n = hist[j];
      if (n > 0) hist[j] = atomicAdd(&p.c.cursor[kbase + j], n);
    }
    __syncthreads();
    for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
      const int key = inv_key(p, e, false);
      if (key >= 0) p.c.entries[atomicAdd(&hist[key], 1)] = static_cast<uint32_t>(e);
    }
  }
}

// Inverse index for key sets too large for a shared-memory histogram.
// Thread order: slot-major, then group, then query, so lanes of a warp read the
// same slot of consecutive queries -- hot blocks (a sink, the previous block)
// collapse into one aggregated atomic per warp.
template <bool SCATTER>
__global__ void inv_index_kernel(const InvParams p) {
  const int64_t total = p.nq * p.H_kv * p.kk;
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t - threadIdx.x < total;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    int64_t key = -1;
    uint32_t slot = 0;
    if (t < total) {
      const int s = static_cast<int>(t / (p.nq * p.H_kv));
      const int64_t rem = t % (p.nq * p.H_kv);
      const int r = static_cast<int>(rem / p.nq);
      const int64_t il = rem % p.nq;
      const int64_t i = p.q0 + il;
      const int32_t b = p.idx[(i * p.H_kv + r) * p.kk + s];
      const int2 sq = seq_of(p.qinfo, i);
      const int64_t b_i = (i - sq.x) / p.B_k;
      if (b < -1 || b >= p.B) {
        if (!SCATTER) report(p.status, DEV_ERR_BAD_INDEX, 40, static_cast<int>(i), b);
      } else if (b >= 0 && b <= b_i) {
        key = ((il / p.Cw) * p.H_kv + r) * p.B + sq.y + b;
        slot = static_cast<uint32_t>((il * p.H_kv + r) * p.kk + s);
      }
    }
    const unsigned active = __ballot_sync(0xFFFFFFFFu, key >= 0);
    if (key >= 0) {
      const unsigned peers = __match_any_sync(active, key);
      const int leader = __ffs(peers) - 1;
      const int lane = threadIdx.x & 31;
      const int rank = __popc(peers & ((1u << lane) - 1));
      if (!SCATTER) {
        if (lane == leader) atomicAdd(&p.c.counts[key], __popc(peers));
      } else {
        int base = 0;
        if (lane == leader) base = atomicAdd(&p.c.cursor[key], __popc(peers));
        base = __shfl_sync(peers, base, leader);
        p.c.entries[base + rank] = slot;
      }
    }
  }
}

// Exclusive scan of (count, tiles) pairs over a block of kScanBlockKeys keys:
// per thread kScanPerThread consecutive keys, warp shuffles, then the warp
// totals.  Returns the thread's exclusive prefix and the block total.
__device__ __forceinline__ void block_scan2(int32_t a, int32_t b, int32_t* ex_a, int32_t* ex_b,
                                            int32_t* tot_a, int32_t* tot_b) {
  __shared__ int32_t ws[2][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int32_t x = a, y = b;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t u = __shfl_up_sync(0xFFFFFFFFu, x, o);
    const int32_t v = __shfl_up_sync(0xFFFFFFFFu, y, o);
    if (lane >= o) {
      x += u;
      y += v;
    }
  }
  if (lane == 31) {
    ws[0][w] = x;
    ws[1][w] = y;
  }
  __syncthreads();
  if (w == 0) {
    const int nw = blockDim.x >> 5;
    int32_t s = lane < nw ? ws[0][lane] : 0, t = lane < nw ? ws[1][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t u = __shfl_up_sync(0xFFFFFFFFu, s, o);
      const int32_t v = __shfl_up_sync(0xFFFFFFFFu, t, o);
      if (lane >= o) {
        s += u;
        t += v;
      }
    }
    ws[0][lane] = s;
    ws[1][lane] = t;
  }
  __syncthreads();
  *ex_a = x - a + (w > 0 ? ws[0][w - 1] : 0);
  *ex_b = y - b + (w > 0 ? ws[1][w - 1] : 0);
  *tot_a = ws[0][31];
  *tot_b = ws[1][31];
  __syncthreads();
}

__device__ __forceinline__ int32_t tiles_of(int32_t count, int Tq) { return (count + Tq - 1) / Tq; }

// Scan, pass 1: per block of keys, the total count and the total tiles.
__global__ void __launch_bounds__(kScanThreads) inv_scan_reduce_kernel(const InvParams p,
                                                                        int64_t nkeys) {
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kScanBlockKeys + threadIdx.x * kScanPerThread;
  int32_t a = 0, b = 0;
#pragma unroll
  for (int j = 0; j < kScanPerThread; ++j)
    if (k0 + j < nkeys) {
      const int32_t c = p.c.counts[k0 + j];
      a += c;
      b += tiles_of(c, p.Tq);
    }
  int32_t ea, eb, ta, tb;
  block_scan2(a, b, &ea, &eb, &ta, &tb);
  if (threadIdx.x == 0) {
    p.c.block_sums[2 * blockIdx.x] = ta;
    p.c.block_sums[2 * blockIdx.x + 1] = tb;
  }
}

// Scan, pass 2 (one block): exclusive scan of the block totals in place, and
// the grand totals.
__global__ void __launch_bounds__(kScanThreads) inv_scan_top_kernel(const InvParams p,
                                                                     int64_t nkeys, int nblocks) {
  int32_t carry_a = 0, carry_b = 0;
  for (int base = 0; base < nblocks; base += kScanThreads) {
    const int g = base + threadIdx.x;
    const int32_t a = g < nblocks ? p.c.block_sums[2 * g] : 0;
    const int32_t b = g < nblocks ? p.c.block_sums[2 * g + 1] : 0;
    int32_t ea, eb, ta, tb;
    block_scan2(a, b, &ea, &eb, &ta, &tb);
    if (g < nblocks) {
      p.c.block_sums[2 * g] = carry_a + ea;
      p.c.block_sums[2 * g + 1] = carry_b + eb;
    }
    carry_a += ta;
    carry_b += tb;
  }
  if (threadIdx.x == 0) {
    p.c.offsets[nkeys] = carry_a;
    p.c.tile_off[nkeys] = carry_b;
    p.c.n_tiles[0] = carry_b;
  }
}

// Scan, pass 3: each key's list offset, scatter cursor and first tile.
__global__ void __launch_bounds__(kScanThreads) inv_scan_apply_kernel(const InvParams p,
                                                                       int64_t nkeys) {
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kScanBlockKeys + threadIdx.x * kScanPerThread;
  int32_t cnt[kScanPerThread];
  int32_t a = 0, b = 0;
#pragma unroll
  for (int j = 0; j < kScanPerThread; ++j) {
    cnt[j] = k0 + j < nkeys ? p.c.counts[k0 + j] : 0;
    a += cnt[j];
    b += tiles_of(cnt[j], p.Tq);
  }
  int32_t ea, eb, ta, tb;
  block_scan2(a, b, &ea, &eb, &ta, &tb);
  int32_t run_a = p.c.block_sums[2 * blockIdx.x] + ea;
  int32_t run_b = p.c.block_sums[2 * blockIdx.x + 1] + eb;
#pragma unroll
  for (int j = 0; j < kScanPerThread; ++j)
    if (k0 + j < nkeys) {
      p.c.offsets[k0 + j] = run_a;
      p.c.cursor[k0 + j] = run_a;
      p.c.tile_off[k0 + j] = run_b;
      run_a += cnt[j];
      run_b += tiles_of(cnt[j], p.Tq);
    }
}

// Per tile: (key, first entry, queries, the key's end tile), one thread per
// tile (a hot key has thousands of tiles).
__global__ void __launch_bounds__(256) inv_tile_meta_kernel(const InvParams p, int64_t nkeys) {
  const int n_tiles = p.c.n_tiles[0];
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < n_tiles; t += gridDim.x * blockDim.x) {
    int64_t lo = 0, hi = nkeys;  // tile_off[lo] <= t < tile_off[hi]
    while (hi - lo > 1) {
      const int64_t mid = (lo + hi) >> 1;
      if (p.c.tile_off[mid] <= t) lo = mid;
      else hi = mid;
    }
    const int32_t t0 = p.c.tile_off[lo], t1 = p.c.tile_off[lo + 1];
    const int32_t o0 = p.c.offsets[lo], o1 = p.c.offsets[lo + 1];
    const int32_t first = o0 + (t - t0) * p.Tq;
    p.c.tile_meta[t] = make_int4(static_cast<int>(lo), first, min(p.Tq, o1 - first), t1);
  }
}

// The inverse index's launch shape: a shared-memory histogram of one
// window's keys per CTA when it fits (up to 4 CTAs per SM), else the
// global-atomic kernels.
cudaError_t inv_setup(int64_t nlocal, int sms, size_t* hist_bytes, int* hist_ctas) {
  *hist_bytes = sizeof(int32_t) * static_cast<size_t>(nlocal);
  *hist_ctas = sms;
  if (*hist_bytes > kMaxHistBytes) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(inv_index_smem_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(*hist_bytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(inv_index_smem_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(*hist_bytes));
  if (e != cudaSuccess) return e;
  const size_t per_sm = 200 * 1024 / (*hist_bytes + 1024);
  *hist_ctas = sms * static_cast<int>(per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm));
  return cudaSuccess;
}

// Count -> scan -> scatter of one chunk's inverse index (counts zeroed before).
void launch_inv_index(const InvParams& ip, size_t hist_bytes, int hist_ctas, int sms,
                      cudaStream_t stream) {
  const int64_t total = ip.nq * ip.H_kv * ip.kk;
  const int64_t nkeys = static_cast<int64_t>(ip.W) * ip.H_kv * ip.B;
  const int nblocks = static_cast<int>(scan_blocks(nkeys));
  const bool smem_path = hist_bytes <= kMaxHistBytes;
  // the histogram grid: whole windows of CTAs
  const int cpw = (hist_ctas + ip.W - 1) / ip.W;
  const int hgrid = cpw * ip.W;
  int blocks = static_cast<int>((total + 255) / 256);
  if (blocks > sms * 16) blocks = sms * 16;
  prof_begin("inv_count", stream);
  if (smem_path) inv_index_smem_kernel<false><<<hgrid, 512, hist_bytes, stream>>>(ip);
  else inv_index_kernel<false><<<blocks, 256, 0, stream>>>(ip);
  prof_end(stream);
  prof_begin("inv_scan", stream);
  inv_scan_reduce_kernel<<<nblocks, kScanThreads, 0, stream>>>(ip, nkeys);
  inv_scan_top_kernel<<<1, kScanThreads, 0, stream>>>(ip, nkeys, nblocks);
  inv_scan_apply_kernel<<<nblocks, kScanThreads, 0, stream>>>(ip, nkeys);
  inv_tile_meta_kernel<<<sms * 4, 256, 0, stream>>>(ip, nkeys);
  prof_end(stream);
  prof_begin("inv_scatter", stream);
  if (smem_path) inv_index_smem_kernel<true><<<hgrid, 512, hist_bytes, stream>>>(ip);
  else inv_index_kernel<true><<<blocks, 256, 0, stream>>>(ip);
  prof_end(stream);
}

// ------------------------------------------------------------------ step 2 --
struct P1Params {
  int64_t q0;
  int q4d;  // 1: one 4-D TMA box per gathered query ([d-chunk][head] rows, 8 heads)
  int H_q, H_kv, B_k, kk, G, R, Tq;
  int B;          // blocks of the sequence (of all sequences, numbered globally)
  int64_t nkeys;  // (window, group, block) keys
  const int32_t* blk_row;  // first token of each global block; null: block b at b * B_k
  float scale_log2;  // softmax scale * log2(e)
  float scale;
  ChunkBufs c;
  DevStatus* status;
};

constexpr int kP1Threads = 512;  // 16 warps, four warpgroups
constexpr int kIR = 8;           // tile-info ring depth (tiles in flight, producer to epilogue)
constexpr int kNS = 2;           // S/P and O buffers in TMEM
// Registers per thread of each warpgroup after the split at kernel start
// (launched with 128 each: 104 + 56 + 2 x 176 = 4 x 128).
constexpr int kRegEpi = 104, kRegCtl = 56, kRegSoftmax = 176;
static_assert(kRegEpi + kRegCtl + 2 * kRegSoftmax <= 4 * 128, "register split above the launch");

template <int D_H, int B_K>
struct P1Shape {
  static constexpr int Q_BYTES = kRowsPerTile * D_H * 2;  // one gathered Q tile
  static constexpr int K_BYTES = B_K * D_H * 2;
  static constexpr int V_BYTES = B_K * D_H * 2;
  static constexpr int NKV = 2;  // K/V slots: the next block lands while the current one is used
  // what the Q ring may take of the 227 KB: minus 1 KB of alignment slack and
  // 2 KB for the tile-info ring and the barriers
  static constexpr int BUDGET = 227 * 1024 - 1024 - 2048;
  static constexpr int QS_FIT = (BUDGET - NKV * (K_BYTES + V_BYTES)) / Q_BYTES;
  static constexpr int QS = QS_FIT > 6 ? 6 : QS_FIT;  // Q ring depth
  static_assert(QS >= 2, "two Q stages must fit");
  static constexpr int DCH = D_H / 64;                // 128-byte chunks along d
  // TMEM columns: S/P buffer b at 128 b, O buffer b at 256 + 128 b
  static constexpr uint32_t TM_S = 0, TM_O = 256;
};

constexpr int kMaxTq = 16;  // queries per tile (128 rows / at least 8 rows per query)

struct TileInfo {
  int r, b, len, gen;  // group, block, queries in the tile, K/V generation
  int jb;              // the block's first token
  uint32_t slot[kMaxTq];  // each query's output slot
  int qi[kMaxTq];         // each query's position i
};

__device__ __forceinline__ int find_key(const int32_t* tile_off, int64_t nkeys, int t) {
  int64_t lo = 0, hi = nkeys;  // tile_off[lo] <= t < tile_off[hi]
  while (hi - lo > 1) {
    const int64_t mid = (lo + hi) >> 1;
    if (tile_off[mid] <= t) lo = mid;
    else hi = mid;
  }
  return static_cast<int>(lo);
}

// Phase 1.  Each CTA owns a contiguous range of tiles; tiles of one (group,
// block) key come in long runs there, so a K/V block stays in its shared
// slot for the whole run; the next run's block loads into the other slot
// meanwhile.  Gathered Q tiles stream through a ring whose stage frees as
// soon as S = Q K^T has been computed.
//   warpgroup 0 (warps 0-3)    epilogue: O (TMEM) -> fp16 partial in HBM
//   warpgroup 1: warp 4        producer (lane q issues query q's TMA box)
//                warp 5        MMA issuer (lane 0) and TMEM owner
//   warpgroups 2, 3            softmax, together on every tile (two warps per
//                              TMEM lane quarter, 16 lanes each)
// TMEM: two S/P buffers (columns 0-255) and two O buffers (256-511), so S of
// the next tile is computed while the softmax works on this one, and the
// tensor core never writes the columns the epilogue is reading.  The softmax reads S, writes
// P = exp(S - m) / l as bf16 over the stage's first B_K/2 columns, and
// O = P V takes P straight from TMEM (tcgen05.mma with A in tensor memory).
// P is normalised, so O needs no rescaling and the epilogue only converts
// and stores it; the softmax writes each row's LSE.
template <int D_H, int B_K>
__global__ void __launch_bounds__(kP1Threads, 1)
    attn_phase1_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const P1Params p) {
  using SH = P1Shape<D_H, B_K>;
  constexpr int QS = SH::QS, NKV = SH::NKV;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;                      // [QS] gathered Q tiles
  uint8_t* sKV = sQ + QS * SH::Q_BYTES;    // [NKV] K block, then V block
  TileInfo* info = reinterpret_cast<TileInfo*>(sKV + NKV * (SH::K_BYTES + SH::V_BYTES));
  uint64_t* bars = reinterpret_cast<uint64_t*>(info + kIR);
  uint64_t* q_full = bars;              // [QS] gathered Q landed
  uint64_t* q_empty = q_full + QS;      // [QS] S of the stage's tile computed
  uint64_t* kv_full = q_empty + QS;     // [NKV] K/V block landed
  uint64_t* kv_empty = kv_full + NKV;   // [NKV] last O = P V of the block's run finished
  uint64_t* i_full = kv_empty + NKV;    // [kIR] tile info written
  uint64_t* i_empty = i_full + kIR;     // [kIR] the tile's epilogue is done
  uint64_t* s_full = i_empty + kIR;     // [kNS] S in TMEM
  uint64_t* p_full = s_full + kNS;      // [kNS] P in TMEM
  uint64_t* o_full = p_full + kNS;      // [kNS] O in TMEM
  uint64_t* o_empty = o_full + kNS;     // [kNS] O read
  uint64_t* fin = o_empty + kNS;        // every MMA of the CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    for (int j = 0; j < NKV; ++j) {
      mbar_init(&kv_full[j], 1);
      mbar_init(&kv_empty[j], 1);
    }
    for (int j = 0; j < kIR; ++j) {
      mbar_init(&i_full[j], 1);
      mbar_init(&i_empty[j], 4);  // the four epilogue warps
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 8);   // the eight softmax warps
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 4);  // the four epilogue warps
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = p.c.n_tiles[0];
  // contiguous tile range of this CTA (tiles are equal-sized units of work;
  // a hot block's list is split over several CTAs)
  const int t_beg = static_cast<int>(static_cast<int64_t>(n_tiles) * blockIdx.x / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(n_tiles) * (blockIdx.x + 1) / gridDim.x);
  const int my_tiles = t_end - t_beg;
  auto tile_of = [&](int n) { return t_beg + n; };
  const int per_q = p.H_kv * p.kk;
  const int wg = warp >> 2;

  if (wg == 1) {
    regs_dec<kRegCtl>();
    if (warp == 4) {
      // ----------------------------------------------------- TMA producer --
      if (lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
      }
      // per tile: (key, first entry, queries, end tile of the key), loaded two
      // tiles ahead; the tile's slots one tile ahead
      auto meta_of = [&](int n) -> int4 {
        return n < my_tiles ? p.c.tile_meta[tile_of(n)] : make_int4(-1, 0, 0, 0);
      };
      int4 meta_next = meta_of(0), meta_next2 = meta_of(1);
      uint32_t next_slot = 0;
      if (my_tiles > 0 && lane < meta_next.z) next_slot = p.c.entries[meta_next.y + lane];
      // K/V generations: a generation is a run of this CTA's tiles with one
      // key; generation g lives in slot g % NKV.  A second cursor finds where
      // the next generation starts so its block loads as soon as its slot is
      // free (one generation ahead), not when its first tile comes up.
      int la_n = 0, la_key = meta_next.x;  // start and key of generation `loaded`
      int la_end = meta_next.w;            // end tile of la_key
      int loaded = 0;                      // generations whose load was issued
      auto advance_la = [&]() {
        // the first tile after la_n whose key differs from la_key: the
        // tile where la_key's list ends
        la_n += la_end - tile_of(la_n);
        if (la_n < my_tiles) {
          const int4 m = meta_of(la_n);
          la_key = m.x;
          la_end = m.w;
        }
      };
      auto load_kv = [&](int g, int k) {
        const int slot = g % NKV;
        const int r = (k / p.B) % p.H_kv, b = k % p.B;
        uint8_t* sK = sKV + slot * (SH::K_BYTES + SH::V_BYTES);
        uint8_t* sV = sK + SH::K_BYTES;
        if (lane == 0) mbar_arrive_expect_tx(&kv_full[slot], SH::K_BYTES + SH::V_BYTES);
        __syncwarp();
        if (lane < SH::DCH) {
          const int row = p.blk_row != nullptr ? p.blk_row[b] : b * B_K;
          tma_load_3d(sK + lane * B_K * 128, &tm_k, &kv_full[slot], lane * 64, r, row);
          tma_load_3d(sV + lane * B_K * 128, &tm_v, &kv_full[slot], lane * 64, r, row);
        }
      };
      int kv_key = -1, kvgen = 0;
      for (int n = 0; n < my_tiles; ++n) {
        const int cur_key = meta_next.x, len = meta_next.z;
        const uint32_t myslot = next_slot;
        const int r = (cur_key / p.B) % p.H_kv, b = cur_key % p.B;
        // the next tile's slots and the metadata of the one after: their
        // latency hides behind the waits below
        meta_next = meta_next2;
        next_slot = (n + 1 < my_tiles && lane < meta_next.z) ? p.c.entries[meta_next.y + lane] : 0u;
        meta_next2 = meta_of(n + 2);
        const bool new_kv = cur_key != kv_key;
        const int gen = new_kv ? kvgen : kvgen - 1;
        const int is = n % kIR, qs = n % QS;
        if (!mbar_wait(&i_empty[is], ((n / kIR) & 1) ^ 1, abort_flag, p.status, 50)) break;
        TileInfo& ti = info[is];
        if (lane < len) {
          ti.slot[lane] = myslot;
          ti.qi[lane] = static_cast<int>(p.q0 + myslot / per_q);
        }
        if (lane == 0) {
          ti.r = r;
          ti.b = b;
          ti.len = len;
          ti.gen = gen;
          ti.jb = p.blk_row != nullptr ? p.blk_row[b] : b * B_K;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&i_full[is]);
        if (!mbar_wait(&q_empty[qs], ((n / QS) & 1) ^ 1, abort_flag, p.status, 52)) break;
        if (lane == 0) mbar_arrive_expect_tx(&q_full[qs], len * p.R * D_H * 2);
        __syncwarp();
        const int h0 = p.G >= 8 ? r * p.G : (r * p.G / 8) * 8;
        if (lane < len) {
          const int i = static_cast<int>(p.q0 + myslot / per_q);
          uint8_t* dst = sQ + qs * SH::Q_BYTES;
          if (p.q4d) {
            // query-major: [query][d-chunk][8 heads x 128 B]
            tma_load_4d(dst + lane * 8 * D_H * 2, &tm_q, &q_full[qs], 0, h0, 0, i);
          } else {
            // chunk-major: [d-chunk][query rows x 128 B]
#pragma unroll
            for (int c = 0; c < SH::DCH; ++c)
              tma_load_3d(dst + c * kRowsPerTile * 128 + lane * p.R * 128, &tm_q, &q_full[qs],
                          c * 64, h0, i);
          }
        }
        if (new_kv) {
          kv_key = cur_key;
          ++kvgen;
        }
        // load every generation up to the one after this tile's: a
        // generation's slot is free once every tile of generation g - NKV
        // finished O = P V (waited for only when this tile needs it)
        bool stop = false;
        while (loaded <= gen + 1 && la_n < my_tiles) {
          const bool need = loaded <= gen;
          if (loaded >= NKV) {
            uint64_t* eb = &kv_empty[loaded % NKV];
            const uint32_t par = ((loaded / NKV) - 1) & 1;
            if (need) {
              if (!mbar_wait(eb, par, abort_flag, p.status, 51)) {
                stop = true;
                break;
              }
            } else if (!__all_sync(0xFFFFFFFFu, mbar_test_wait(eb, par))) {
              break;
            }
          }
          load_kv(loaded, la_key);
          ++loaded;
          advance_la();
        }
        if (stop) break;
      }
    } else if (warp == 5 && lane == 0) {
      // ------------------------------------------------------ MMA issuer --
      // S(n) goes before O(n-1) when tile n's rows and K block have landed,
      // so the tensor core works while the softmax of n-1 finishes; else
      // O(n-1) goes first so it never waits behind a gather (or behind a K/V
      // block that can only load once O(n-1) frees its slot).  S(n) reuses
      // the S/P buffer of tile n-2, whose O MMA (reading P there) was issued
      // before it: tcgen05.mma ops of one thread run in issue order.
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, B_K, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D_H, 0, 1);
      const uint32_t q_sbo = p.q4d ? 8 * D_H * 2 : 1024;  // between 8-row groups
      const uint32_t q_cstep = p.q4d ? 8 * 128 : kRowsPerTile * 128;  // between d-chunks
      int kv_ready = -1;  // highest K/V generation known to have landed
      auto prep = [&](int n, int* gen) -> bool {
        if (!mbar_wait(&i_full[n % kIR], (n / kIR) & 1, abort_flag, p.status, 60)) return false;
        *gen = info[n % kIR].gen;
        return true;
      };
      auto s_ready = [&](int n, int gen) -> bool {
        return mbar_test_wait(&q_full[n % QS], (n / QS) & 1) &&
               (gen <= kv_ready || mbar_test_wait(&kv_full[gen % NKV], (gen / NKV) & 1));
      };
      auto issue_s = [&](int n, int gen) -> bool {
        if (!mbar_wait(&q_full[n % QS], (n / QS) & 1, abort_flag, p.status, 61)) return false;
        if (gen > kv_ready) {
          if (!mbar_wait(&kv_full[gen % NKV], (gen / NKV) & 1, abort_flag, p.status, 62))
            return false;
          kv_ready = gen;
        }
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + (n % QS) * SH::Q_BYTES);
        const uint32_t k_base = smem_u32(sKV + (gen % NKV) * (SH::K_BYTES + SH::V_BYTES));
        const uint32_t tS = tmem_base + (n % kNS) * 128 + SH::TM_S;
#pragma unroll
        for (int c = 0; c < SH::DCH; ++c)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint64_t ad = umma_desc(q_base + c * q_cstep + s * 32, 16, q_sbo, SW_128B);
            const uint64_t bd = umma_desc(k_base + c * B_K * 128 + s * 32, 16, 1024, SW_128B);
            umma_bf16(tS, ad, bd, idesc_s, (c | s) != 0);
          }
        umma_commit(&s_full[n % kNS]);
        umma_commit(&q_empty[n % QS]);
        return true;
      };
      auto issue_o = [&](int m, int gen, bool last_of_gen) -> bool {
        if (!mbar_wait(&p_full[m % kNS], (m / kNS) & 1, abort_flag, p.status, 63)) return false;
        if (!mbar_wait(&o_empty[m % kNS], ((m / kNS) & 1) ^ 1, abort_flag, p.status, 64))
          return false;
        tc_fence_after();
        const uint32_t v_base =
            smem_u32(sKV + (gen % NKV) * (SH::K_BYTES + SH::V_BYTES) + SH::K_BYTES);
        const uint32_t tP = tmem_base + (m % kNS) * 128 + SH::TM_S;
        const uint32_t tO = tmem_base + SH::TM_O + (m % kNS) * 128;
#pragma unroll
        for (int ks = 0; ks < B_K / 16; ++ks) {
          // V: MN-major (d contiguous); 16 keys = two 8-key groups = 2048 B
          const uint64_t bd = umma_desc(v_base + ks * 2048, B_K * 128, 1024, SW_128B);
          umma_bf16_ts(tO, tP + ks * 8, bd, idesc_o, ks != 0);
        }
        umma_commit(&o_full[m % kNS]);
        if (last_of_gen) umma_commit(&kv_empty[gen % NKV]);
        return true;
      };
      if (my_tiles > 0) {
        int gprev = 0;
        bool ok = prep(0, &gprev) && issue_s(0, gprev);
        for (int n = 1; ok && n < my_tiles; ++n) {
          int gn = 0;
          if (!prep(n, &gn)) break;
          const bool last = gn != gprev;
          if (s_ready(n, gn)) ok = issue_s(n, gn) && issue_o(n - 1, gprev, last);
          else ok = issue_o(n - 1, gprev, last) && issue_s(n, gn);
          gprev = gn;
        }
        if (ok) issue_o(my_tiles - 1, gprev, true);
      }
      // every MMA of this CTA must be done before TMEM is released
      umma_commit(fin);
      mbar_wait(fin, 0, nullptr, p.status, 69);
    }
  } else if (wg == 0) {
    // -------------------------------------------------------- epilogue --
    regs_dec<kRegEpi>();
    const int row = warp * 32 + lane;  // warp w reads TMEM lanes 32w .. 32w+31
    const int q_local = row / p.R;
    const int hrow = row - q_local * p.R;
    for (int n = 0; n < my_tiles; ++n) {
      const int is = n % kIR;
      if (!mbar_wait(&i_full[is], (n / kIR) & 1, abort_flag, p.status, 70)) break;
      if (!mbar_wait(&o_full[n % kNS], (n / kNS) & 1, abort_flag, p.status, 71)) break;
      tc_fence_after();
      const TileInfo& ti = info[is];
      const int goff = p.G >= 8 ? 0 : (ti.r * p.G) % 8;  // group's first head in the box
      const bool useful = q_local < ti.len && hrow >= goff && hrow < goff + p.G;
      const int g = hrow - goff;
      const uint32_t slot = useful ? ti.slot[q_local] : 0u;
      // partial layout [slot][d/8][g][8]: for one d/8 the G heads of a query
      // are G consecutive 16-byte pieces, so a warp's stores cover whole
      // 128-byte lines
      __half* dst = p.c.part_o + static_cast<int64_t>(slot) * p.G * D_H + g * 8;
      const uint32_t tO =
          tmem_base + SH::TM_O + (n % kNS) * 128 + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
      for (int hc = 0; hc < D_H / 64; ++hc) {
        uint32_t ra[32], rb[32];
        tmem_ld32(tO + hc * 64, ra);
        tmem_ld32(tO + hc * 64 + 32, rb);
        tmem_wait_ld();
        if (hc == D_H / 64 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty[n % kNS]);
        }
        if (useful) {
#pragma unroll
          for (int j = 0; j < 64; j += 8) {
            const uint32_t* src = j < 32 ? &ra[j] : &rb[j - 32];
            uint4 w;
            __half2 a0 = __floats2half2_rn(__uint_as_float(src[0]), __uint_as_float(src[1]));
            __half2 a1 = __floats2half2_rn(__uint_as_float(src[2]), __uint_as_float(src[3]));
            __half2 a2 = __floats2half2_rn(__uint_as_float(src[4]), __uint_as_float(src[5]));
            __half2 a3 = __floats2half2_rn(__uint_as_float(src[6]), __uint_as_float(src[7]));
            w.x = *reinterpret_cast<uint32_t*>(&a0);
            w.y = *reinterpret_cast<uint32_t*>(&a1);
            w.z = *reinterpret_cast<uint32_t*>(&a2);
            w.w = *reinterpret_cast<uint32_t*>(&a3);
            const int d8 = (hc * 64 + j) >> 3;
            // written once and read once by the merge: stream past L2 so the
            // gathered Q rows stay cached
            __stcs(reinterpret_cast<uint4*>(dst + d8 * p.G * 8), w);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&i_empty[is]);
    }
  } else {
    // ---------------------------------------------------------- softmax --
    regs_inc<kRegSoftmax>();
    // All eight warps take every tile: warps w and w + 4 share TMEM lane
    // quarter w % 4, the first taking its lanes 0-15, the second 16-31.  A
    // thread holds two rows (lanes lo = base + lane/4 and hi = lo + 8) x the
    // row's keys 8r + 2c, 8r + 2c + 1 (c = lane % 4, r = 0 .. B_K/8 - 1), so
    // a row's reductions take two shuffles across its four threads, and the
    // bf16 pair of keys (8r + 2c, 8r + 2c + 1) is exactly P column 4r + c of
    // the 16x128b store shape.
    const int half = (warp - 8) >> 2;
    const int quarter = warp & 3;
    const int gq = lane >> 2, cq = lane & 3;
    const int lane0 = quarter * 32 + half * 16;  // first TMEM lane of this warp
    const int rowA = lane0 + gq, rowB = rowA + 8;
    const int qA = rowA / p.R, hA = rowA - qA * p.R;
    const int qB = rowB / p.R, hB = rowB - qB * p.R;
    // When S of tile n + 1 is already complete, its TMEM load is issued
    // before P of tile n is stored, so the load latency overlaps the store
    // and the barrier hand-off.  (It is never waited for there: the MMA
    // warp may be waiting for this P before it issues S of n + 1.)
    uint32_t v[B_K / 2];  // v[4r + 0/1]: row A, keys 8r + 2c + 0/1; v[4r + 2/3]: row B
    auto s_landed = [&](int n) -> bool {
      const bool mine = mbar_test_wait(&i_full[n % kIR], (n / kIR) & 1) &&
                        mbar_test_wait(&s_full[n % kNS], (n / kNS) & 1);
      return __all_sync(0xFFFFFFFFu, mine);  // every lane saw both phases complete
    };
    auto load_s = [&](int n, bool landed) -> bool {
      const int st = n % kNS;
      if (!landed) {
        if (!mbar_wait(&i_full[n % kIR], (n / kIR) & 1, abort_flag, p.status, 80)) return false;
        if (!mbar_wait(&s_full[st], (n / kNS) & 1, abort_flag, p.status, 81)) return false;
      }
      tc_fence_after();
      const uint32_t tS = tmem_base + st * 128 + SH::TM_S + (static_cast<uint32_t>(lane0) << 16);
#pragma unroll
      for (int h = 0; h < B_K / 64; ++h) {
        uint32_t t32[32];
        tmem_ld_16x256b_x8(tS + h * 64, t32);
#pragma unroll
        for (int j = 0; j < 32; ++j) v[h * 32 + j] = t32[j];
      }
      return true;
    };
    bool ok = my_tiles > 0 && load_s(0, false);
    for (int n = 0; ok && n < my_tiles; ++n) {
      const int st = n % kNS, is = n % kIR;
      const uint32_t tS = tmem_base + st * 128 + SH::TM_S + (static_cast<uint32_t>(lane0) << 16);
      const TileInfo& ti = info[is];
      const int goff = p.G >= 8 ? 0 : (ti.r * p.G) % 8;  // group's first head in the box
      const bool liveA = qA < ti.len, liveB = qB < ti.len;
      const uint32_t slotA = liveA ? ti.slot[qA] : 0u;
      const uint32_t slotB = liveB ? ti.slot[qB] : 0u;
      // a padding row (past the tile's queries) is never masked
      const int iA = liveA ? ti.qi[qA] : INT_MAX;
      const int iB = liveB ? ti.qi[qB] : INT_MAX;
      const int jb = ti.jb;  // the block's first key
      tmem_wait_ld();
      if (jb + B_K - 1 > (iA < iB ? iA : iB)) {  // a query's own block: j <= i
#pragma unroll
        for (int r = 0; r < B_K / 8; ++r)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = jb + 8 * r + 2 * cq + e;
            if (j > iA) v[4 * r + e] = __float_as_uint(-INFINITY);
            if (j > iB) v[4 * r + 2 + e] = __float_as_uint(-INFINITY);
          }
      }
      float mA = -INFINITY, mB = -INFINITY;
#pragma unroll
      for (int r = 0; r < B_K / 8; ++r) {
        mA = fmax3(mA, __uint_as_float(v[4 * r]), __uint_as_float(v[4 * r + 1]));
        mB = fmax3(mB, __uint_as_float(v[4 * r + 2]), __uint_as_float(v[4 * r + 3]));
      }
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        mA = fmaxf(mA, __shfl_xor_sync(0xFFFFFFFFu, mA, o));
        mB = fmaxf(mB, __shfl_xor_sync(0xFFFFFFFFu, mB, o));
      }
      const float msA = mA * p.scale_log2, msB = mB * p.scale_log2;
      float lA0 = 0.0f, lA1 = 0.0f, lB0 = 0.0f, lB1 = 0.0f;
#pragma unroll
      for (int r = 0; r < B_K / 8; ++r) {
        const float a0 = ex2_ftz(fmaf(__uint_as_float(v[4 * r]), p.scale_log2, -msA));
        const float a1 = ex2_ftz(fmaf(__uint_as_float(v[4 * r + 1]), p.scale_log2, -msA));
        const float b0 = ex2_ftz(fmaf(__uint_as_float(v[4 * r + 2]), p.scale_log2, -msB));
        const float b1 = ex2_ftz(fmaf(__uint_as_float(v[4 * r + 3]), p.scale_log2, -msB));
        lA0 += a0;
        lA1 += a1;
        lB0 += b0;
        lB1 += b1;
        v[4 * r] = __float_as_uint(a0);
        v[4 * r + 1] = __float_as_uint(a1);
        v[4 * r + 2] = __float_as_uint(b0);
        v[4 * r + 3] = __float_as_uint(b1);
      }
      float lA = lA0 + lA1, lB = lB0 + lB1;
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        lA += __shfl_xor_sync(0xFFFFFFFFu, lA, o);
        lB += __shfl_xor_sync(0xFFFFFFFFu, lB, o);
      }
      const float invA = 1.0f / lA, invB = 1.0f / lB;
      // P / l as bf16 pairs: the pair of keys (8r + 2c, 8r + 2c + 1) is P
      // column 4r + c
      uint32_t pk[B_K / 4];
#pragma unroll
      for (int r = 0; r < B_K / 8; ++r) {
        __nv_bfloat162 xa = __floats2bfloat162_rn(__uint_as_float(v[4 * r]) * invA,
                                                  __uint_as_float(v[4 * r + 1]) * invA);
        __nv_bfloat162 xb = __floats2bfloat162_rn(__uint_as_float(v[4 * r + 2]) * invB,
                                                  __uint_as_float(v[4 * r + 3]) * invB);
        pk[2 * r] = *reinterpret_cast<uint32_t*>(&xa);
        pk[2 * r + 1] = *reinterpret_cast<uint32_t*>(&xb);
      }
      const bool more = n + 1 < my_tiles;
      const bool early = more && s_landed(n + 1);
      if (early) load_s(n + 1, true);  // into v: this tile's values are all in pk now
      // P over the stage's first B_K / 2 columns (its S was read)
#pragma unroll
      for (int h = 0; h < B_K / 64; ++h) {
        uint32_t q16[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) q16[j] = pk[h * 16 + j];
        tmem_st_16x128b_x8(tS + h * 32, q16);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
      if (cq == 0) {
        if (liveA && hA >= goff && hA < goff + p.G)
          p.c.part_lse[static_cast<int64_t>(slotA) * p.G + (hA - goff)] = mA * p.scale + logf(lA);
        if (liveB && hB >= goff && hB < goff + p.G)
          p.c.part_lse[static_cast<int64_t>(slotB) * p.G + (hB - goff)] = mB * p.scale + logf(lB);
      }
      if (more && !early) ok = load_s(n + 1, false);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ step 3 --
struct MergeParams {
  const int32_t* idx;
  __nv_bfloat16* o;
  float* lse;
  int64_t q0, nq;
  int H_q, H_kv, kk, G, B_k;
  const int2* qinfo;  // packed sequences (per token), or null
  ChunkBufs c;
};

// LSE-weighted merge of each row's partials (split-K softmax normalisation).
// W warps per (query, group); a lane owns E = min(32, G*D_H/(32*W)) consecutive
// outputs of one head.  Per slot a lane needs its head's LSE (4 B) and E fp16
// partial values: all of a row's LSEs are fetched at once, then the partial
// rows four slots at a time, so each warp keeps several KB of loads in flight.
// A warp writes its G x D_H output block as contiguous 16-byte pieces.
template <int D_H, int E>
__global__ void __launch_bounds__(256, 2) attn_merge_kernel(const MergeParams p) {
  static_assert(E % 8 == 0 && D_H % E == 0, "lane slice must be whole 16-byte pieces of one head");
  constexpr int V16 = E / 8;  // 16-byte loads per slot
  const int lane = threadIdx.x & 31;
  const int W = (p.G * D_H) / (32 * E);  // warps per (query, group)
  const int64_t gw = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t unit = gw / W;
  if (unit >= p.nq * p.H_kv) return;
  const int wq = static_cast<int>(gw - unit * W);
  const int64_t il = unit / p.H_kv;
  const int r = static_cast<int>(unit - il * p.H_kv);
  const int e0 = (wq * 32 + lane) * E;  // element offset inside the [G, D_H] block
  const int g = e0 / D_H, d0 = e0 - g * D_H;
  const int64_t i = p.q0 + il;
  const int64_t b_i = (i - seq_of(p.qinfo, i).x) / p.B_k;
  const int64_t slot0 = (il * p.H_kv + r) * p.kk;
  int32_t myb = -1;
  if (lane < p.kk) myb = p.idx[(i * p.H_kv + r) * p.kk + lane];
  const unsigned use = __ballot_sync(0xFFFFFFFFu, lane < p.kk && myb >= 0 && myb <= b_i);
  // this lane's head: the largest LSE of its used slots (read again below,
  // from L1, rather than held in registers)
  const float* lse_h = p.c.part_lse + slot0 * p.G + g;
  float m = -INFINITY;
  for (int s = 0; s < p.kk; ++s)
    if ((use >> s) & 1u) m = fmaxf(m, lse_h[s * p.G]);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.0f;
  float wsum = 0.0f;
  // partial layout [slot][d/8][g][8]
  const __half* base = p.c.part_o + slot0 * p.G * D_H + (d0 >> 3) * p.G * 8 + g * 8;
  const int64_t stride = static_cast<int64_t>(p.G) * D_H;  // between slots
  const int cstride = p.G * 8;                              // between d-chunks
#pragma unroll
  for (int s0 = 0; s0 < p.kk; s0 += 4) {
    uint4 x[4][V16];
    float w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int s = s0 + j;
      const bool on = s < p.kk && ((use >> s) & 1u);
      w[j] = on ? __expf(lse_h[s * p.G] - m) : 0.0f;
#pragma unroll
      for (int u = 0; u < V16; ++u)
        x[j][u] = on ? *reinterpret_cast<const uint4*>(base + s * stride + u * cstride)
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      wsum += w[j];
#pragma unroll
      for (int u = 0; u < V16; ++u) {
        const __half2* hv = reinterpret_cast<const __half2*>(&x[j][u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __half22float2(hv[e]);
          acc[u * 8 + 2 * e] = fmaf(w[j], f.x, acc[u * 8 + 2 * e]);
          acc[u * 8 + 2 * e + 1] = fmaf(w[j], f.y, acc[u * 8 + 2 * e + 1]);
        }
      }
    }
  }
  const int h = r * p.G + g;
  __nv_bfloat16* dst = p.o + (i * p.H_q + h) * static_cast<int64_t>(D_H) + d0;
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
#pragma unroll
  for (int u = 0; u < V16; ++u) {
    uint4 o4;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o4);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 t = __floats2bfloat162_rn(acc[u * 8 + 2 * e] * inv, acc[u * 8 + 2 * e + 1] * inv);
      ow[e] = *reinterpret_cast<uint32_t*>(&t);
    }
    *reinterpret_cast<uint4*>(dst + u * 8) = o4;
  }
  if (p.lse != nullptr && d0 == 0) p.lse[i * p.H_q + h] = use ? m + logf(wsum) : -INFINITY;
}

// Merge for G * D_H < 256 outputs per (query, group), where one warp per
// (query, group) would have idle lanes: one thread per 8 consecutive outputs
// of one head; each thread reads its (query, group)'s selection and its
// head's LSEs itself.
template <int D_H>
__global__ void __launch_bounds__(256) attn_merge_small_kernel(const MergeParams p) {
  const int per_unit = p.G * D_H / 8;  // threads per (query, group)
  const int64_t gt = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t unit = gt / per_unit;
  if (unit >= p.nq * p.H_kv) return;
  const int e0 = static_cast<int>(gt - unit * per_unit) * 8;
  const int g = e0 / D_H, d0 = e0 - g * D_H;
  const int64_t il = unit / p.H_kv;
  const int r = static_cast<int>(unit - il * p.H_kv);
  const int64_t i = p.q0 + il;
  const int64_t b_i = (i - seq_of(p.qinfo, i).x) / p.B_k;
  const int64_t slot0 = (il * p.H_kv + r) * p.kk;
  const int32_t* sel = p.idx + (i * p.H_kv + r) * p.kk;
  const float* lse_h = p.c.part_lse + slot0 * p.G + g;
  float m = -INFINITY;
  for (int s = 0; s < p.kk; ++s) {
    const int b = sel[s];
    if (b >= 0 && b <= b_i) m = fmaxf(m, lse_h[s * p.G]);
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
  float wsum = 0.0f;
  // partial layout [slot][d/8][g][8]
  const __half* base = p.c.part_o + slot0 * p.G * D_H + (d0 >> 3) * p.G * 8 + g * 8;
  for (int s = 0; s < p.kk; ++s) {
    const int b = sel[s];
    if (b < 0 || b > b_i) continue;
    const float w = __expf(lse_h[s * p.G] - m);
    wsum += w;
    const uint4 x = *reinterpret_cast<const uint4*>(base + static_cast<int64_t>(s) * p.G * D_H);
    const __half2* hv = reinterpret_cast<const __half2*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(hv[e]);
      acc[2 * e] = fmaf(w, f.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(w, f.y, acc[2 * e + 1]);
    }
  }
  const int h = r * p.G + g;
  const float inv = wsum > 0.0f ? 1.0f / wsum : 0.0f;
  uint4 o4;
  uint32_t* ow = reinterpret_cast<uint32_t*>(&o4);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 t = __floats2bfloat162_rn(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    ow[e] = *reinterpret_cast<uint32_t*>(&t);
  }
  *reinterpret_cast<uint4*>(p.o + (i * p.H_q + h) * static_cast<int64_t>(D_H) + d0) = o4;
  if (p.lse != nullptr && d0 == 0) p.lse[i * p.H_q + h] = wsum > 0.0f ? m + logf(wsum) : -INFINITY;
}

template <int D_H, int B_K>
size_t p1_smem_bytes() {
  using SH = P1Shape<D_H, B_K>;
  return 1024 + SH::QS * SH::Q_BYTES + SH::NKV * (SH::K_BYTES + SH::V_BYTES) +
         kIR * sizeof(TileInfo) + (2 * SH::QS + 2 * SH::NKV + 2 * kIR + 4 * kNS + 1) * 8 + 16;
}

template <int D_H, int B_K>
cudaError_t launch_typed(const AttnLaunch& a, cudaStream_t stream) {
  const int G = a.H_q / a.H_kv;
  const int R = rows_per_query(G);
  const int Tq = kRowsPerTile / R;
  const int64_t B = a.B_tot > 0 ? a.B_tot : (a.N + a.B_k - 1) / a.B_k;
  const int64_t Nc = chunk_len(a.N, a.B_k);
  const int64_t nkeys_max = inv_nkeys(Nc, kWindow, a.H_kv, B);  // per chunk, at most
  size_t need = 0;
  ChunkBufs c = carve(a.ws, Nc, a.H_q, a.H_kv, a.d_h, a.kk, nkeys_max, &need);
  if (need > a.ws_bytes) return cudaErrorInvalidValue;

  CUtensorMap tq, tk, tv;
  int q4d = 0;
  if (R == 8) {
    // (64 d, heads, d-chunk, query): one box = 8 heads x all of d, landing as
    // [d-chunk][head] 128-byte rows
    const uint64_t dims[4] = {64, static_cast<uint64_t>(a.H_q), static_cast<uint64_t>(D_H / 64),
                              static_cast<uint64_t>(a.N)};
    const uint64_t strides[3] = {static_cast<uint64_t>(D_H) * 2, 128,
                                 static_cast<uint64_t>(a.H_q) * D_H * 2};
    const uint32_t box[4] = {64, 8, static_cast<uint32_t>(D_H / 64), 1};
    q4d = make_tmap_bf16(&tq, a.q, 4, dims, strides, box, 128) ? 1 : 0;
  }
  if (!q4d) {
    const uint64_t dims[3] = {static_cast<uint64_t>(D_H), static_cast<uint64_t>(a.H_q),
                              static_cast<uint64_t>(a.N)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D_H) * 2,
                                 static_cast<uint64_t>(a.H_q) * D_H * 2};
    const uint32_t box[3] = {64, static_cast<uint32_t>(R), 1};
    if (!make_tmap_bf16(&tq, a.q, 3, dims, strides, box, 128)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(D_H), static_cast<uint64_t>(a.H_kv),
                              static_cast<uint64_t>(a.N)};
    const uint64_t strides[2] = {static_cast<uint64_t>(D_H) * 2,
                                 static_cast<uint64_t>(a.H_kv) * D_H * 2};
    const uint32_t box[3] = {64, 1, static_cast<uint32_t>(B_K)};
    if (!make_tmap_bf16(&tk, a.k, 3, dims, strides, box, 128)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16(&tv, a.v, 3, dims, strides, box, 128)) return cudaErrorInvalidValue;
  }
  const size_t smem = p1_smem_bytes<D_H, B_K>();
  cudaError_t e = cudaFuncSetAttribute(attn_phase1_kernel<D_H, B_K>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  size_t hist_bytes = 0;
  int hist_grid = 0;
  e = inv_setup(a.H_kv * B, sms, &hist_bytes, &hist_grid);
  if (e != cudaSuccess) return e;

  for (int64_t q0 = 0; q0 < a.N; q0 += Nc) {
    const int64_t nq = (a.N - q0) < Nc ? (a.N - q0) : Nc;
    const int64_t nkeys = inv_nkeys(nq, kWindow, a.H_kv, B);
    e = cudaMemsetAsync(c.counts, 0, sizeof(int32_t) * nkeys, stream);
    if (e != cudaSuccess) return e;
    InvParams ip{};
    ip.idx = a.idx;
    ip.q0 = q0;
    ip.nq = nq;
    ip.H_kv = a.H_kv;
    ip.B_k = a.B_k;
    ip.kk = a.kk;
    ip.B = B;
    ip.qinfo = a.qinfo;
    ip.Tq = Tq;
    ip.Cw = kWindow;
    ip.W = static_cast<int>((nq + kWindow - 1) / kWindow);
    ip.c = c;
    ip.status = a.status;
    launch_inv_index(ip, hist_bytes, hist_grid, sms, stream);

    P1Params pp{};
    pp.q0 = q0;
    pp.q4d = q4d;
    pp.H_q = a.H_q;
    pp.H_kv = a.H_kv;
    pp.B_k = a.B_k;
    pp.kk = a.kk;
    pp.G = G;
    pp.R = R;
    pp.Tq = Tq;
    pp.B = static_cast<int>(B);
    pp.nkeys = nkeys;
    pp.blk_row = a.blk_row;
    pp.scale = a.scale;
    pp.scale_log2 = a.scale * 1.4426950408889634f;
    pp.c = c;
    pp.status = a.status;
    prof_begin("attn_phase1", stream);
    attn_phase1_kernel<D_H, B_K><<<sms, kP1Threads, smem, stream>>>(tq, tk, tv, pp);
    prof_end(stream);

    MergeParams mp{};
    mp.idx = a.idx;
    mp.o = static_cast<__nv_bfloat16*>(a.o);
    mp.lse = a.lse;
    mp.q0 = q0;
    mp.nq = nq;
    mp.H_q = a.H_q;
    mp.H_kv = a.H_kv;
    mp.kk = a.kk;
    mp.G = G;
    mp.B_k = a.B_k;
    mp.qinfo = a.qinfo;
    mp.c = c;
    prof_begin("attn_merge", stream);
    if (G * D_H < 256) {
      const int64_t threads = nq * a.H_kv * (G * D_H / 8);
      const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
      attn_merge_small_kernel<D_H><<<blocks, 256, 0, stream>>>(mp);
    } else {
      const int per_unit = G * D_H / 32;           // outputs per lane with one warp
      const int E = per_unit >= 32 ? 32 : (per_unit >= 16 ? 16 : 8);
      const int W = G * D_H / (32 * E);
      const int64_t warps = nq * a.H_kv * W;
      const unsigned blocks = static_cast<unsigned>((warps * 32 + 255) / 256);
      if (E == 32) attn_merge_kernel<D_H, 32><<<blocks, 256, 0, stream>>>(mp);
      else if (E == 16) attn_merge_kernel<D_H, 16><<<blocks, 256, 0, stream>>>(mp);
      else attn_merge_kernel<D_H, 8><<<blocks, 256, 0, stream>>>(mp);
    }
    prof_end(stream);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------ KL-loss fusion: LSE_idx (Eq. 9) --
// The normaliser of the Index Branch distribution over the selected token
// set, LSE_idx[i, r] = log sum_{j in selected blocks, j <= i} exp(S^idx), as
// each selected block's LSE reduced over the Top-k blocks (review, "4.3 Sparse
// KL Loss Fusion"; notes 5.4).  KV-outer like phase 1: the inverse index lists,
// per (group, block), the selection slots that chose it; a warp takes 16 of
// them (one 16-row mma.sync tile: the slots' index queries against the
// block's K_idx rows, both read straight from L2) and writes each slot's
// block LSE; a second kernel reduces a row's slots.
struct IdxLseParams {
  const __nv_bfloat16* q_idx;  // [N, H_kv, d_idx]
  const __nv_bfloat16* k_idx;  // [N, d_idx]
  int64_t q0, N, nkeys;
  int H_kv, kk, B_k;
  float scale_log2;
  ChunkBufs c;
};

constexpr int kLseTile = 16;  // slots per warp tile (mma.sync M)

// Shared-memory row of one K_idx key in idx_lse_kernel: d_idx bf16 plus 16
// bytes, so the 8 rows an ldmatrix reads fall in distinct bank groups.
template <int D_IDX>
__host__ __device__ constexpr int lse_row_bytes() { return D_IDX * 2 + 16; }
constexpr int kLseWarps = 4;  // warps per CTA of idx_lse_kernel

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                      uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <int D_IDX, int B_K>
__global__ void __launch_bounds__(32 * kLseWarps) idx_lse_kernel(const IdxLseParams p) {
  constexpr int KS = D_IDX / 16;  // k-steps
  constexpr int NT = B_K / 8;     // 8-key n-tiles of a block
  constexpr int ROW = lse_row_bytes<D_IDX>();
  extern __shared__ uint8_t lse_smem[];
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  // this warp's copy of the current block's K_idx rows (one key's run of tiles)
  uint8_t* sk = lse_smem + (threadIdx.x >> 5) * B_K * ROW;
  const uint32_t sk_u32 = smem_u32(sk);
  int staged = -1;
  const int n_tiles = p.c.n_tiles[0];
  const int64_t warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  // a contiguous range of tiles per warp: keys are walked forward
  const int t_beg = static_cast<int>(n_tiles * w / warps);
  const int t_end = static_cast<int>(n_tiles * (w + 1) / warps);
  if (t_beg >= t_end) return;
  const int nb = static_cast<int>(p.nkeys / p.H_kv);
  const int per_q = p.H_kv * p.kk;
  int key = find_key(p.c.tile_off, p.nkeys, t_beg);
  int kend = p.c.tile_off[key + 1];
  for (int tile = t_beg; tile < t_end; ++tile) {
    while (kend <= tile) kend = p.c.tile_off[++key + 1];
    const int r = key / nb, b = key - r * nb;
    if (b != staged) {
      // the block's K_idx rows into shared memory, 16 bytes per lane and
      // step (rows past N as zeros)
      constexpr int CPR = D_IDX / 8;  // 16-byte pieces per row
      __syncwarp();
      for (int c = lane; c < B_K * CPR; c += 32) {
        const int row = c / CPR, col = c - row * CPR;
        const int64_t j = static_cast<int64_t>(b) * B_K + row;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (j < p.N) v = __ldg(reinterpret_cast<const uint4*>(p.k_idx + j * D_IDX) + col);
        *reinterpret_cast<uint4*>(sk + row * ROW + col * 16) = v;
      }
      __syncwarp();
      staged = b;
    }
    const int koff = p.c.offsets[key];
    const int first = koff + (tile - p.c.tile_off[key]) * kLseTile;
    const int len = min(kLseTile, p.c.offsets[key + 1] - first);
    const bool v_lo = g < len, v_hi = g + 8 < len;
    const uint32_t s_lo = v_lo ? p.c.entries[first + g] : 0u;
    const uint32_t s_hi = v_hi ? p.c.entries[first + g + 8] : 0u;
    const int64_t i_lo = p.q0 + s_lo / per_q, i_hi = p.q0 + s_hi / per_q;
    // A: the index queries of rows g and g+8 (zero for rows past the tile)
    const __nv_bfloat16* q_lo = p.q_idx + (i_lo * p.H_kv + r) * D_IDX + 2 * t;
    const __nv_bfloat16* q_hi = p.q_idx + (i_hi * p.H_kv + r) * D_IDX + 2 * t;
    uint32_t qa[KS][4];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = v_lo ? __ldg(reinterpret_cast<const unsigned int*>(q_lo + ks * 16)) : 0u;
      qa[ks][1] = v_hi ? __ldg(reinterpret_cast<const unsigned int*>(q_hi + ks * 16)) : 0u;
      qa[ks][2] = v_lo ? __ldg(reinterpret_cast<const unsigned int*>(q_lo + ks * 16 + 8)) : 0u;
      qa[ks][3] = v_hi ? __ldg(reinterpret_cast<const unsigned int*>(q_hi + ks * 16 + 8)) : 0u;
    }
    // S = Q_idx K_idx^T over the block's keys, B fragments by ldmatrix: the
    // four 8x8 matrices are (keys n, d lo), (keys n, d hi), (keys n+8, d lo),
    // (keys n+8, d hi)
    const int64_t j0 = static_cast<int64_t>(b) * B_K;
    float acc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.0f;
    {
      const int mi = lane >> 3, rr = lane & 7;
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2)
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          const int key_row = n2 * 16 + (mi >> 1) * 8 + rr;
          const int d = ks * 16 + (mi & 1) * 8;
          uint32_t b0, b1, b2, b3;
          ldsm4(sk_u32 + key_row * ROW + d * 2, b0, b1, b2, b3);
          mma_bf16_16816(acc[2 * n2], qa[ks], b0, b1);
          mma_bf16_16816(acc[2 * n2 + 1], qa[ks], b2, b3);
        }
    }
    // the block's LSE for each row, log2 domain: causal rule j <= i
    float m_lo = -INFINITY, m_hi = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t j = j0 + nt * 8 + 2 * t + (e & 1);
        const bool lo = e < 2;
        float x = acc[nt][e] * p.scale_log2;
        if (j > (lo ? i_lo : i_hi)) x = -INFINITY;
        acc[nt][e] = x;
        if (lo) m_lo = fmaxf(m_lo, x);
        else m_hi = fmaxf(m_hi, x);
      }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      m_lo = fmaxf(m_lo, __shfl_xor_sync(0xFFFFFFFFu, m_lo, o));
      m_hi = fmaxf(m_hi, __shfl_xor_sync(0xFFFFFFFFu, m_hi, o));
    }
    float l_lo = 0.0f, l_hi = 0.0f;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      l_lo += exp2f(acc[nt][0] - m_lo) + exp2f(acc[nt][1] - m_lo);
      l_hi += exp2f(acc[nt][2] - m_hi) + exp2f(acc[nt][3] - m_hi);
    }
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
      l_lo += __shfl_xor_sync(0xFFFFFFFFu, l_lo, o);
      l_hi += __shfl_xor_sync(0xFFFFFFFFu, l_hi, o);
    }
    // natural-log LSE of the slot's block (every slot here holds j = i or an
    // earlier block, so m is finite)
    constexpr float kLn2 = 0.6931471805599453f;
    if (t == 0 && v_lo) p.c.part_lse[s_lo] = (m_lo + log2f(l_lo)) * kLn2;
    if (t == 0 && v_hi) p.c.part_lse[s_hi] = (m_hi + log2f(l_hi)) * kLn2;
  }
}

// LSE_idx[i, r]: log-sum-exp of the row's block LSEs over its valid slots.
__global__ void __launch_bounds__(256) idx_lse_combine_kernel(const int32_t* idx, float* lse_idx,
                                                              const IdxLseParams p, int64_t nq) {
  const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (u >= nq * p.H_kv) return;
  const int64_t il = u / p.H_kv;
  const int r = static_cast<int>(u - il * p.H_kv);
  const int64_t i = p.q0 + il;
  const int64_t b_i = i / p.B_k;
  const int32_t* sel = idx + (i * p.H_kv + r) * p.kk;
  const float* part = p.c.part_lse + (il * p.H_kv + r) * p.kk;
  float m = -INFINITY;
  for (int s = 0; s < p.kk; ++s) {
    const int b = sel[s];
    if (b >= 0 && b <= b_i) m = fmaxf(m, part[s]);
  }
  float sum = 0.0f;
  for (int s = 0; s < p.kk; ++s) {
    const int b = sel[s];
    if (b >= 0 && b <= b_i) sum += __expf(part[s] - m);
  }
  lse_idx[i * p.H_kv + r] = sum > 0.0f ? m + logf(sum) : -INFINITY;
}

template <int D_IDX, int B_K>
cudaError_t launch_idx_lse_typed(const IdxLseLaunch& a, cudaStream_t stream) {
  const int64_t B = (a.N + B_K - 1) / B_K;
  const int64_t nkeys = a.H_kv * B;
  const int64_t Nc = chunk_len(a.N, B_K);
  size_t need = 0;
  // the inverse index and one fp32 LSE per slot (a chunk's buffers with G = 1, no partial O)
  ChunkBufs c = carve(a.ws, Nc, a.H_kv, a.H_kv, 0, a.kk, nkeys, &need);
  if (need > a.ws_bytes) return cudaErrorInvalidValue;
  const int sms = num_sms();
  size_t hist_bytes = 0;
  int hist_grid = 0;
  cudaError_t e = inv_setup(nkeys, sms, &hist_bytes, &hist_grid);
  if (e != cudaSuccess) return e;
  const size_t lse_smem = static_cast<size_t>(kLseWarps) * B_K * lse_row_bytes<D_IDX>();
  e = cudaFuncSetAttribute(idx_lse_kernel<D_IDX, B_K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(lse_smem));
  if (e != cudaSuccess) return e;
  // CTAs per SM: the SM's 228 KB of shared memory, 1 KB of it reserved per CTA
  const int lse_ctas = static_cast<int>(228 * 1024 / (lse_smem + 1024));
  for (int64_t q0 = 0; q0 < a.N; q0 += Nc) {
    const int64_t nq = (a.N - q0) < Nc ? (a.N - q0) : Nc;
    e = cudaMemsetAsync(c.counts, 0, sizeof(int32_t) * nkeys, stream);
    if (e != cudaSuccess) return e;
    InvParams ip{};
    ip.idx = a.idx;
    ip.q0 = q0;
    ip.nq = nq;
    ip.H_kv = a.H_kv;
    ip.B_k = B_K;
    ip.kk = a.kk;
    ip.B = B;
    ip.Tq = kLseTile;
    ip.Cw = static_cast<int>(Nc);  // one window: keys (group, block)
    ip.W = 1;
    ip.c = c;
    ip.status = a.status;
    launch_inv_index(ip, hist_bytes, hist_grid, sms, stream);
    IdxLseParams lp;
    lp.q_idx = static_cast<const __nv_bfloat16*>(a.q_idx);
    lp.k_idx = static_cast<const __nv_bfloat16*>(a.k_idx);
    lp.q0 = q0;
    lp.N = a.N;
    lp.nkeys = nkeys;
    lp.H_kv = a.H_kv;
    lp.kk = a.kk;
    lp.B_k = B_K;
    lp.scale_log2 = a.scale * 1.4426950408889634f;
    lp.c = c;
    prof_begin("idx_lse", stream);
    idx_lse_kernel<D_IDX, B_K><<<sms * lse_ctas, 32 * kLseWarps, lse_smem, stream>>>(lp);
    prof_end(stream);
    prof_begin("idx_lse_combine", stream);
    idx_lse_combine_kernel<<<static_cast<unsigned>((nq * a.H_kv + 255) / 256), 256, 0, stream>>>(
        a.idx, a.lse_idx, lp, nq);
    prof_end(stream);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// ------------------------------------------------- backward of Eq. 8 --
// Gradients of the Main Branch with the selection fixed (the Index Branch
// is not differentiated through its Top-k; review §四, "Dynamic load
// balancing", and §五 4.3 place the backward beside the forward's KV-outer
// schedule).  With P = softmax over the selected keys j <= i (recomputed from
// the forward's LSE), D = rowsum(dO * O) and dS = P (dO V^T - D):
//   dQ = scale dS K,   dK = scale dS^T Q,   dV = P^T dO.
// Both kernels walk the forward's inverse-index tiles (one (group, block)
// key, 128 rows = 128/G queries x the group's G heads):
//   bwd_dq_kernel    rows per warp: S, P, dP, dS and the tile's dQ partial
//                    per (row, slot), fp32, summed per row afterwards;
//   bwd_dkdv_kernel  keys per warp: dK and dV of the warp's 16 keys kept in
//                    registers over a unit of consecutive tiles (mostly one
//                    key), units taken from a global atomic counter so hot
//                    blocks spread over the SMs; each unit adds its sums to
//                    fp32 accumulators with vector atomics.
constexpr int kBwdThreads = 256;  // 8 warps
constexpr int kBwdRows = 128;     // rows (query, head) per tile
constexpr int kBwdUnit = 32;      // tiles per work unit of the dK/dV kernel

struct BwdParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dO;
  const float* lse;  // [N, H_q] natural log (the forward's)
  const float* D;    // [N, H_q] rowsum(dO * O)
  int64_t N, q0;
  int H_q, H_kv, G, kk, B;
  float scale, scale_log2;
  ChunkBufs c;
  float* dq_part;  // [chunk slots, G, d_h]
  float* dk_acc;   // [N, H_kv, d_h]
  float* dv_acc;
  int* work;
  DevStatus* status;
};

// Byte offset of (row, d) in a [ROWS][D] bf16 tile held as D/64 boxes of
// ROWS 128-byte rows, 16-byte chunks XOR (row % 8): the 8 rows an ldmatrix
// reads fall in distinct bank groups.
template <int ROWS>
__device__ __forceinline__ uint32_t bsw(int row, int d) {
  return static_cast<uint32_t>((d >> 6) * (ROWS * 128) + row * 128 +
                               ((((d >> 3) & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// wait until at most N of this thread's most recent groups are pending
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Per-row scalars of the tile in shared memory.
struct BwdRows {
  float lse2[kBwdRows];  // LSE * log2(e); +inf for padding rows (P = 0)
  float Drow[kBwdRows];
  int qi[kBwdRows];      // query position; -1 for padding rows
  uint32_t slot[kBwdRows];
  int64_t src[kBwdRows];  // row index i * H_q + h of Q / dO
};

template <int D_H, int B_K>
struct BwdSmem {
  static constexpr int Q_BYTES = kBwdRows * D_H * 2;
  static constexpr int K_BYTES = B_K * D_H * 2;
  // two stages of the tile's Q and dO rows (the next tile's land while the
  // current one computes), one K/V block
  static constexpr size_t bytes() {
    return 128 + 4 * Q_BYTES + 2 * K_BYTES + 2 * sizeof(BwdRows);
  }
};

// The tile's per-row scalars (threads 0..127); the caller synchronises
// before bwd_issue_rows reads them.
__device__ __forceinline__ void bwd_row_scalars(const BwdParams& p, int4 meta, int r,
                                                BwdRows* rows) {
  const int per_q = p.H_kv * p.kk;
  const int t = threadIdx.x;
  if (t < kBwdRows) {
    const int qq = t / p.G, g = t - (t / p.G) * p.G;
    if (qq < meta.z) {
      const uint32_t e = p.c.entries[meta.y + qq];
      const int64_t i = p.q0 + e / per_q;
      const int64_t s = i * p.H_q + r * p.G + g;
      rows->slot[t] = e;
      rows->qi[t] = static_cast<int>(i);
      rows->src[t] = s;
      rows->lse2[t] = p.lse[s] * 1.4426950408889634f;
      rows->Drow[t] = p.D[s];
    } else {
      rows->slot[t] = 0;
      rows->qi[t] = -1;
      rows->src[t] = -1;
      rows->lse2[t] = INFINITY;
      rows->Drow[t] = 0.f;
    }
  }
}

// The tile's Q and dO rows by 16-byte async copies (padding rows
// zero-filled), one commit group.
template <int D_H>
__device__ __forceinline__ void bwd_issue_rows(const BwdParams& p, const BwdRows* rows,
                                               uint8_t* sQ, uint8_t* sdO) {
  constexpr int CPR = D_H / 8;  // 16-byte chunks per row
  const int t = threadIdx.x;
  const uint32_t q_base = smem_u32(sQ), g_base = smem_u32(sdO);
  for (int c = t; c < kBwdRows * CPR; c += kBwdThreads) {
    const int row = c / CPR, ch = c - row * CPR;
    const int64_t s = rows->src[row];
    const bool ok = s >= 0;
    const int64_t off = (ok ? s : 0) * D_H + ch * 8;
    cp_async16(q_base + bsw<kBwdRows>(row, ch * 8), p.q + off, ok);
    cp_async16(g_base + bsw<kBwdRows>(row, ch * 8), p.dO + off, ok);
  }
  cp_async_commit();
}

// Start loading tile `tile` into stage st: its scalars, then its rows.
template <int D_H>
__device__ __forceinline__ void bwd_prefetch(const BwdParams& p, int tile, BwdRows* rows,
                                             uint8_t* sQ, uint8_t* sdO) {
  const int4 meta = p.c.tile_meta[tile];
  bwd_row_scalars(p, meta, (meta.x / p.B) % p.H_kv, rows);
  __syncthreads();
  bwd_issue_rows<D_H>(p, rows, sQ, sdO);
}

// The K and V rows of block b of group r (rows past N zero-filled).
template <int D_H, int B_K>
__device__ __forceinline__ void bwd_load_kv(const BwdParams& p, int r, int b, uint8_t* sK,
                                            uint8_t* sV) {
  constexpr int CPR = D_H / 8;
  const uint32_t k_base = smem_u32(sK), v_base = smem_u32(sV);
  for (int c = threadIdx.x; c < B_K * CPR; c += kBwdThreads) {
    const int key = c / CPR, ch = c - key * CPR;
    const int64_t j = static_cast<int64_t>(b) * B_K + key;
    const bool ok = j < p.N;
    const int64_t off = ((ok ? j : 0) * p.H_kv + r) * D_H + ch * 8;
    cp_async16(k_base + bsw<B_K>(key, ch * 8), p.k + off, ok);
    cp_async16(v_base + bsw<B_K>(key, ch * 8), p.v + off, ok);
  }
  cp_async_commit();
}

// dQ: each CTA walks a contiguous range of tiles; warp w owns rows
// [16w, 16w + 16) of every tile.
template <int D_H, int B_K>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dq_kernel(const BwdParams p) {
  using SM = BwdSmem<D_H, B_K>;
  constexpr int NT = B_K / 8, KS = D_H / 16, DT = D_H / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  // stage s: Q rows at smem + 2s Q_BYTES, dO rows right after
  auto sQs = [&](int st) { return smem + st * 2 * SM::Q_BYTES; };
  auto sdOs = [&](int st) { return smem + st * 2 * SM::Q_BYTES + SM::Q_BYTES; };
  uint8_t* sK = smem + 4 * SM::Q_BYTES;
  uint8_t* sV = sK + SM::K_BYTES;
  BwdRows* rows_s = reinterpret_cast<BwdRows*>(sV + SM::K_BYTES);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const int n_tiles = p.c.n_tiles[0];
  const int t_beg = static_cast<int>(static_cast<int64_t>(n_tiles) * blockIdx.x / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(n_tiles) * (blockIdx.x + 1) / gridDim.x);
  int kv_key = -1;
  if (t_beg < t_end) bwd_prefetch<D_H>(p, t_beg, &rows_s[0], sQs(0), sdOs(0));
  for (int tile = t_beg; tile < t_end; ++tile) {
    const int st = (tile - t_beg) & 1;
    const int4 meta = p.c.tile_meta[tile];
    const int r = (meta.x / p.B) % p.H_kv, b = meta.x % p.B;
    if (meta.x != kv_key) {  // every warp finished the previous tile (barrier below)
      bwd_load_kv<D_H, B_K>(p, r, b, sK, sV);
      kv_key = meta.x;
    }
    // the next tile's rows land while this one computes
    if (tile + 1 < t_end) {
      bwd_prefetch<D_H>(p, tile + 1, &rows_s[st ^ 1], sQs(st ^ 1), sdOs(st ^ 1));
      cp_async_wait_group<1>();
    } else {
      cp_async_wait_group<0>();
    }
    __syncthreads();
    const BwdRows* rows = &rows_s[st];
    const uint32_t qb = smem_u32(sQs(st)), gb = smem_u32(sdOs(st)), kb = smem_u32(sK),
                   vb = smem_u32(sV);
    // S = Q K^T and dP = dO V^T for the warp's 16 rows
    float sacc[NT][4], pacc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[n][e] = pacc[n][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t qa[4], ga[4];
      const int arow = warp * 16 + (mi & 1) * 8 + rr, ad = ks * 16 + (mi >> 1) * 8;
      ldsm_x4(qb + bsw<kBwdRows>(arow, ad), qa[0], qa[1], qa[2], qa[3]);
      ldsm_x4(gb + bsw<kBwdRows>(arow, ad), ga[0], ga[1], ga[2], ga[3]);
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2) {
        const int key = n2 * 16 + (mi >> 1) * 8 + rr, d = ks * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + bsw<B_K>(key, d), b0, b1, b2, b3);
        mma_bf16_16816(sacc[2 * n2], qa, b0, b1);
        mma_bf16_16816(sacc[2 * n2 + 1], qa, b2, b3);
        ldsm_x4(vb + bsw<B_K>(key, d), b0, b1, b2, b3);
        mma_bf16_16816(pacc[2 * n2], ga, b0, b1);
        mma_bf16_16816(pacc[2 * n2 + 1], ga, b2, b3);
      }
    }
    // P (causal within the block), dS = P (dP - D), packed as the A operand
    const int rA = warp * 16 + g, rB = rA + 8;
    const int iA = rows->qi[rA], iB = rows->qi[rB];
    const float lA = rows->lse2[rA], lB = rows->lse2[rB];
    const float DA = rows->Drow[rA], DB = rows->Drow[rB];
    const int jb = b * B_K;
    uint32_t da[NT / 2][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      float ds[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = jb + n * 8 + 2 * t4 + (e & 1);
        const int i = e < 2 ? iA : iB;
        const float pr = (i < 0 || j > i) ? 0.f
                                          : exp2f(sacc[n][e] * p.scale_log2 - (e < 2 ? lA : lB));
        ds[e] = pr * (pacc[n][e] - (e < 2 ? DA : DB));
      }
      da[n >> 1][(n & 1) * 2 + 0] = pack_bf16(ds[0], ds[1]);
      da[n >> 1][(n & 1) * 2 + 1] = pack_bf16(ds[2], ds[3]);
    }
    // dQ partial = dS K (k = the block's keys)
    float qacc[DT][4];
#pragma unroll
    for (int n = 0; n < DT; ++n) qacc[n][0] = qacc[n][1] = qacc[n][2] = qacc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < B_K / 16; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < DT / 2; ++n2) {
        const int key = ks * 16 + (mi & 1) * 8 + rr, d = n2 * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(kb + bsw<B_K>(key, d), b0, b1, b2, b3);
        mma_bf16_16816(qacc[2 * n2], da[ks], b0, b1);
        mma_bf16_16816(qacc[2 * n2 + 1], da[ks], b2, b3);
      }
    }
    if (iA >= 0) {
      float* dst = p.dq_part + (static_cast<int64_t>(rows->slot[rA]) * p.G + rA % p.G) * D_H;
#pragma unroll
      for (int n = 0; n < DT; ++n)
        *reinterpret_cast<float2*>(dst + n * 8 + 2 * t4) =
            make_float2(qacc[n][0] * p.scale, qacc[n][1] * p.scale);
    }
    if (iB >= 0) {
      float* dst = p.dq_part + (static_cast<int64_t>(rows->slot[rB]) * p.G + rB % p.G) * D_H;
#pragma unroll
      for (int n = 0; n < DT; ++n)
        *reinterpret_cast<float2*>(dst + n * 8 + 2 * t4) =
            make_float2(qacc[n][2] * p.scale, qacc[n][3] * p.scale);
    }
    __syncthreads();  // the tile's shared memory is free
  }
}

// dK, dV: units of kBwdUnit consecutive tiles from a global counter; warp w
// owns keys [16w, 16w + 16) of the block (B_K / 16 warps compute) and keeps
// their dK, dV in registers while the unit stays on one key.
template <int D_H, int B_K, int RH>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_dkdv_kernel(const BwdParams p) {
  using SM = BwdSmem<D_H, B_K>;
  constexpr int KS = D_H / 16, DT = D_H / 8, NR = RH / 8;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                             ~static_cast<uintptr_t>(127));
  // stage s: Q rows at smem + 2s Q_BYTES, dO rows right after
  auto sQs = [&](int st) { return smem + st * 2 * SM::Q_BYTES; };
  auto sdOs = [&](int st) { return smem + st * 2 * SM::Q_BYTES + SM::Q_BYTES; };
  uint8_t* sK = smem + 4 * SM::Q_BYTES;
  uint8_t* sV = sK + SM::K_BYTES;
  BwdRows* rows_s = reinterpret_cast<BwdRows*>(sV + SM::K_BYTES);
  __shared__ int s_unit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const bool keys_warp = warp * 16 < B_K;
  const int n_tiles = p.c.n_tiles[0];
  float kacc[DT][4], vacc[DT][4];
  auto zero = [&]() {
#pragma unroll
    for (int n = 0; n < DT; ++n)
#pragma unroll
      for (int e = 0; e < 4; ++e) kacc[n][e] = vacc[n][e] = 0.f;
  };
  // add the warp's sums for (group r, block b) to the fp32 accumulators
  auto flush = [&](int r, int b) {
    if (!keys_warp) return;
    const int64_t jA = static_cast<int64_t>(b) * B_K + warp * 16 + g, jB = jA + 8;
#pragma unroll
    for (int n = 0; n < DT; ++n) {
      const int d = n * 8 + 2 * t4;
      if (jA < p.N) {
        const int64_t o = (jA * p.H_kv + r) * D_H + d;
        atomicAdd(reinterpret_cast<float2*>(p.dk_acc + o),
                  make_float2(kacc[n][0] * p.scale, kacc[n][1] * p.scale));
        atomicAdd(reinterpret_cast<float2*>(p.dv_acc + o), make_float2(vacc[n][0], vacc[n][1]));
      }
      if (jB < p.N) {
        const int64_t o = (jB * p.H_kv + r) * D_H + d;
        atomicAdd(reinterpret_cast<float2*>(p.dk_acc + o),
                  make_float2(kacc[n][2] * p.scale, kacc[n][3] * p.scale));
        atomicAdd(reinterpret_cast<float2*>(p.dv_acc + o), make_float2(vacc[n][2], vacc[n][3]));
      }
    }
  };
  for (;;) {
    if (threadIdx.x == 0) s_unit = atomicAdd(p.work, 1);
    __syncthreads();
    const int t0 = s_unit * kBwdUnit;
    __syncthreads();  // every thread has read s_unit
    if (t0 >= n_tiles) break;
    const int t1 = t0 + kBwdUnit < n_tiles ? t0 + kBwdUnit : n_tiles;
    int cur = -1, cr = 0, cb = 0;
    zero();
    bwd_prefetch<D_H>(p, t0, &rows_s[0], sQs(0), sdOs(0));
    for (int tile = t0; tile < t1; ++tile) {
      const int st = (tile - t0) & 1;
      const int4 meta = p.c.tile_meta[tile];
      const int r = (meta.x / p.B) % p.H_kv, b = meta.x % p.B;
      if (meta.x != cur) {
        if (cur >= 0) flush(cr, cb);
        zero();
        cur = meta.x;
        cr = r;
        cb = b;
        bwd_load_kv<D_H, B_K>(p, r, b, sK, sV);
      }
      if (tile + 1 < t1) {
        bwd_prefetch<D_H>(p, tile + 1, &rows_s[st ^ 1], sQs(st ^ 1), sdOs(st ^ 1));
        cp_async_wait_group<1>();
      } else {
        cp_async_wait_group<0>();
      }
      __syncthreads();
      const BwdRows* rows = &rows_s[st];
      if (keys_warp) {
        const uint32_t qb = smem_u32(sQs(st)), gb = smem_u32(sdOs(st)), kb = smem_u32(sK),
                       vb = smem_u32(sV);
        const int jA = b * B_K + warp * 16 + g, jB = jA + 8;  // the thread's two keys
#pragma unroll 1
        for (int r0 = 0; r0 < kBwdRows; r0 += RH) {
          // S^T = K Q^T and dP^T = V dO^T for the warp's keys x RH rows
          float st[NR][4], dpt[NR][4];
#pragma unroll
          for (int n = 0; n < NR; ++n)
#pragma unroll
            for (int e = 0; e < 4; ++e) st[n][e] = dpt[n][e] = 0.f;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            uint32_t ka[4], va[4];
            const int arow = warp * 16 + (mi & 1) * 8 + rr, ad = ks * 16 + (mi >> 1) * 8;
            ldsm_x4(kb + bsw<B_K>(arow, ad), ka[0], ka[1], ka[2], ka[3]);
            ldsm_x4(vb + bsw<B_K>(arow, ad), va[0], va[1], va[2], va[3]);
#pragma unroll
            for (int n2 = 0; n2 < NR / 2; ++n2) {
              const int row = r0 + n2 * 16 + (mi >> 1) * 8 + rr, d = ks * 16 + (mi & 1) * 8;
              uint32_t b0, b1, b2, b3;
              ldsm_x4(qb + bsw<kBwdRows>(row, d), b0, b1, b2, b3);
              mma_bf16_16816(st[2 * n2], ka, b0, b1);
              mma_bf16_16816(st[2 * n2 + 1], ka, b2, b3);
              ldsm_x4(gb + bsw<kBwdRows>(row, d), b0, b1, b2, b3);
              mma_bf16_16816(dpt[2 * n2], va, b0, b1);
              mma_bf16_16816(dpt[2 * n2 + 1], va, b2, b3);
            }
          }
          // P^T and dS^T, packed as A operands (k = rows)
          uint32_t pa[NR / 2][4], da[NR / 2][4];
#pragma unroll
          for (int n = 0; n < NR; ++n) {
            float pv[4], dv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = r0 + n * 8 + 2 * t4 + (e & 1);
              const int i = rows->qi[row];
              const int j = e < 2 ? jA : jB;
              pv[e] = (i < 0 || j > i) ? 0.f : exp2f(st[n][e] * p.scale_log2 - rows->lse2[row]);
              dv[e] = pv[e] * (dpt[n][e] - rows->Drow[row]);
            }
            pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(pv[0], pv[1]);
            pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(pv[2], pv[3]);
            da[n >> 1][(n & 1) * 2 + 0] = pack_bf16(dv[0], dv[1]);
            da[n >> 1][(n & 1) * 2 + 1] = pack_bf16(dv[2], dv[3]);
          }
          // dV += P^T dO, dK += dS^T Q (k = rows; B by transposing loads)
#pragma unroll
          for (int ks = 0; ks < RH / 16; ++ks) {
#pragma unroll
            for (int n2 = 0; n2 < DT / 2; ++n2) {
              const int row = r0 + ks * 16 + (mi & 1) * 8 + rr, d = n2 * 16 + (mi >> 1) * 8;
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(gb + bsw<kBwdRows>(row, d), b0, b1, b2, b3);
              mma_bf16_16816(vacc[2 * n2], pa[ks], b0, b1);
              mma_bf16_16816(vacc[2 * n2 + 1], pa[ks], b2, b3);
              ldsm_x4_t(qb + bsw<kBwdRows>(row, d), b0, b1, b2, b3);
              mma_bf16_16816(kacc[2 * n2], da[ks], b0, b1);
              mma_bf16_16816(kacc[2 * n2 + 1], da[ks], b2, b3);
            }
          }
        }
      }
      __syncthreads();  // the tile's shared memory is free
    }
    if (cur >= 0) flush(cr, cb);
  }
}

// D[i, h] = rowsum(dO * O): one warp per row.
template <int D_H>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* dO,
                                                       const __nv_bfloat16* o, int64_t rows,
                                                       float* D) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float acc = 0.f;
  for (int d = lane * 2; d < D_H; d += 64) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dO + row * D_H + d));
    const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + row * D_H + d));
    acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
  }
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, m);
  if (lane == 0) D[row] = acc;
}

// dQ[i, h] = sum of the row's partials over its used slots (bf16 out); one
// warp per (query, head), lane l owning d = 4l .. 4l + 3 (D_H = 128) or
// 2l .. 2l + 1 (D_H = 64).
template <int D_H>
__global__ void __launch_bounds__(256) bwd_dq_sum_kernel(const BwdParams p, const int32_t* idx,
                                                         int64_t nq, int B_k,
                                                         __nv_bfloat16* dq) {
  constexpr int E = D_H / 32;
  const int64_t u = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (u >= nq * p.H_q) return;
  const int64_t il = u / p.H_q;
  const int h = static_cast<int>(u - il * p.H_q);
  const int r = h / p.G, g = h - r * p.G;
  const int64_t i = p.q0 + il;
  const int64_t b_i = i / B_k;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int s = 0; s < p.kk; ++s) {
    const int b = idx[(i * p.H_kv + r) * p.kk + s];
    if (b < 0 || b > b_i) continue;
    const float* src = p.dq_part + (((il * p.H_kv + r) * p.kk + s) * p.G + g) * D_H + lane * E;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += src[e];
  }
  __nv_bfloat16* dst = dq + (i * p.H_q + h) * D_H + lane * E;
#pragma unroll
  for (int e = 0; e < E; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(acc[e], acc[e + 1]);
}

__global__ void __launch_bounds__(256) bwd_convert_kernel(const float* a, const float* b,
                                                          int64_t n, __nv_bfloat16* ya,
                                                          __nv_bfloat16* yb) {
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  if (t >= n) return;
  *reinterpret_cast<__nv_bfloat162*>(ya + t) = __floats2bfloat162_rn(a[t], a[t + 1]);
  *reinterpret_cast<__nv_bfloat162*>(yb + t) = __floats2bfloat162_rn(b[t], b[t + 1]);
}

// Workspace of the backward: the inverse index and fp32 dQ partials of a
// chunk of Nc queries, then D, the dK/dV accumulators and the work counter.
struct BwdBufs {
  ChunkBufs c;
  float* D;
  float* dk_acc;
  float* dv_acc;
  int* work;
};
int64_t bwd_chunk_len(int64_t N, int B_k) { return chunk_len(N < kMaxChunk / 2 ? N : kMaxChunk / 2, B_k); }

BwdBufs bwd_carve(void* ws, int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk,
                  size_t* total) {
  BwdBufs w;
  const int64_t B = (N + B_k - 1) / B_k;
  const int64_t Nc = bwd_chunk_len(N, B_k);
  const int G = H_q / H_kv;
  size_t used = 0;
  // the fp32 partials take the room of fp16 ones of twice the head dim
  w.c = carve(ws, Nc, H_q, H_kv, 2 * d_h, kk, inv_nkeys(Nc, kWindow, H_kv, B), &used);
  (void)G;
  uint8_t* base = static_cast<uint8_t*>(ws);
  auto take = [&](size_t bytes) {
    uint8_t* r = base ? base + used : nullptr;
    used += align256(bytes);
    return r;
  };
  w.D = reinterpret_cast<float*>(take(sizeof(float) * N * H_q));
  w.dk_acc = reinterpret_cast<float*>(take(sizeof(float) * N * H_kv * d_h));
  w.dv_acc = reinterpret_cast<float*>(take(sizeof(float) * N * H_kv * d_h));
  w.work = reinterpret_cast<int*>(take(256));
  *total = used;
  return w;
}

template <int D_H, int B_K>
cudaError_t launch_bwd_typed(const BwdLaunch& a, cudaStream_t stream) {
  const int G = a.H_q / a.H_kv;
  const int Tq = kBwdRows / G;
  const int64_t B = (a.N + a.B_k - 1) / a.B_k;
  size_t need = 0;
  BwdBufs w = bwd_carve(a.ws, a.N, a.H_q, a.H_kv, D_H, a.B_k, a.kk, &need);
  if (need > a.ws_bytes) return cudaErrorInvalidValue;
  const int64_t Nc = bwd_chunk_len(a.N, a.B_k);
  using SM = BwdSmem<D_H, B_K>;
  const size_t smem = SM::bytes();
  constexpr int RH = D_H == 128 ? 32 : 64;  // rows per pass of the dK/dV kernel (registers)
  cudaError_t e = cudaFuncSetAttribute(bwd_dq_kernel<D_H, B_K>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D_H, B_K, RH>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  size_t hist_bytes = 0;
  int hist_grid = 0;
  e = inv_setup(a.H_kv * B, sms, &hist_bytes, &hist_grid);
  if (e != cudaSuccess) return e;
  const int64_t kv_elems = a.N * a.H_kv * D_H;
  e = cudaMemsetAsync(w.dk_acc, 0, sizeof(float) * kv_elems, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.dv_acc, 0, sizeof(float) * kv_elems, stream);
  if (e != cudaSuccess) return e;
  {
    const int64_t rows = a.N * a.H_q;
    prof_begin("bwd_prep", stream);
    bwd_prep_kernel<D_H><<<static_cast<unsigned>((rows * 32 + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.dO), static_cast<const __nv_bfloat16*>(a.o), rows,
        w.D);
    prof_end(stream);
  }
  BwdParams bp{};
  bp.q = static_cast<const __nv_bfloat16*>(a.q);
  bp.k = static_cast<const __nv_bfloat16*>(a.k);
  bp.v = static_cast<const __nv_bfloat16*>(a.v);
  bp.dO = static_cast<const __nv_bfloat16*>(a.dO);
  bp.lse = a.lse;
  bp.D = w.D;
  bp.N = a.N;
  bp.H_q = a.H_q;
  bp.H_kv = a.H_kv;
  bp.G = G;
  bp.kk = a.kk;
  bp.B = static_cast<int>(B);
  bp.scale = a.scale;
  bp.scale_log2 = a.scale * 1.4426950408889634f;
  bp.c = w.c;
  bp.dq_part = reinterpret_cast<float*>(w.c.part_o);
  bp.dk_acc = w.dk_acc;
  bp.dv_acc = w.dv_acc;
  bp.work = w.work;
  bp.status = a.status;
  for (int64_t q0 = 0; q0 < a.N; q0 += Nc) {
    const int64_t nq = (a.N - q0) < Nc ? (a.N - q0) : Nc;
    const int64_t nkeys = inv_nkeys(nq, kWindow, a.H_kv, B);
    e = cudaMemsetAsync(w.c.counts, 0, sizeof(int32_t) * nkeys, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(w.work, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    InvParams ip{};
    ip.idx = a.idx;
    ip.q0 = q0;
    ip.nq = nq;
    ip.H_kv = a.H_kv;
    ip.B_k = a.B_k;
    ip.kk = a.kk;
    ip.B = B;
    ip.Tq = Tq;
    ip.Cw = kWindow;
    ip.W = static_cast<int>((nq + kWindow - 1) / kWindow);
    ip.c = w.c;
    ip.status = a.status;
    launch_inv_index(ip, hist_bytes, hist_grid, sms, stream);
    bp.q0 = q0;
    prof_begin("bwd_dq", stream);
    bwd_dq_kernel<D_H, B_K><<<sms, kBwdThreads, smem, stream>>>(bp);
    prof_end(stream);
    prof_begin("bwd_dkdv", stream);
    bwd_dkdv_kernel<D_H, B_K, RH><<<sms, kBwdThreads, smem, stream>>>(bp);
    prof_end(stream);
    const int64_t warps = nq * a.H_q;
    prof_begin("bwd_dq_sum", stream);
    bwd_dq_sum_kernel<D_H><<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, stream>>>(
        bp, a.idx, nq, a.B_k, static_cast<__nv_bfloat16*>(a.dq));
    prof_end(stream);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  prof_begin("bwd_convert", stream);
  bwd_convert_kernel<<<static_cast<unsigned>((kv_elems / 2 + 255) / 256), 256, 0, stream>>>(
      w.dk_acc, w.dv_acc, kv_elems, static_cast<__nv_bfloat16*>(a.dk),
      static_cast<__nv_bfloat16*>(a.dv));
  prof_end(stream);
  return cudaGetLastError();
}

}  // namespace

size_t idx_lse_workspace_bytes(int64_t N, int H_kv, int B_k, int kk) {
  const int64_t B = (N + B_k - 1) / B_k;
  size_t total = 0;
  carve(nullptr, chunk_len(N, B_k), H_kv, H_kv, 0, kk, H_kv * B, &total);
  return total;
}

cudaError_t launch_idx_lse(const IdxLseLaunch& a, cudaStream_t s) {
  if (a.d_idx == 64 && a.B_k == 128) return launch_idx_lse_typed<64, 128>(a, s);
  if (a.d_idx == 64 && a.B_k == 64) return launch_idx_lse_typed<64, 64>(a, s);
  if (a.d_idx == 128 && a.B_k == 128) return launch_idx_lse_typed<128, 128>(a, s);
  if (a.d_idx == 128 && a.B_k == 64) return launch_idx_lse_typed<128, 64>(a, s);
  if (a.d_idx == 32 && a.B_k == 128) return launch_idx_lse_typed<32, 128>(a, s);
  if (a.d_idx == 32 && a.B_k == 64) return launch_idx_lse_typed<32, 64>(a, s);
  return cudaErrorInvalidValue;
}

size_t attn_workspace_bytes(int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk,
                            int64_t B_tot) {
  const int64_t B = B_tot > 0 ? B_tot : (N + B_k - 1) / B_k;
  size_t total = 0;
  const int64_t Nc = chunk_len(N, B_k);
  carve(nullptr, Nc, H_q, H_kv, d_h, kk, inv_nkeys(Nc, kWindow, H_kv, B), &total);
  return total;
}

cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t s) {
  if (a.d_h == 128 && a.B_k == 128) return launch_typed<128, 128>(a, s);
  if (a.d_h == 128 && a.B_k == 64) return launch_typed<128, 64>(a, s);
  if (a.d_h == 64 && a.B_k == 128) return launch_typed<64, 128>(a, s);
  if (a.d_h == 64 && a.B_k == 64) return launch_typed<64, 64>(a, s);
  return cudaErrorInvalidValue;
}

size_t attn_bwd_workspace_bytes(int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk) {
  size_t total = 0;
  bwd_carve(nullptr, N, H_q, H_kv, d_h, B_k, kk, &total);
  return total;
}

cudaError_t launch_sparse_attn_bwd(const BwdLaunch& a, cudaStream_t s) {
  if (a.d_h == 128 && a.B_k == 128) return launch_bwd_typed<128, 128>(a, s);
  if (a.d_h == 128 && a.B_k == 64) return launch_bwd_typed<128, 64>(a, s);
  if (a.d_h == 64 && a.B_k == 128) return launch_bwd_typed<64, 128>(a, s);
  if (a.d_h == 64 && a.B_k == 64) return launch_bwd_typed<64, 64>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace msa
