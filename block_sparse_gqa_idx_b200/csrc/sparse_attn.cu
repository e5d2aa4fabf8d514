// sparse_attn.cu -- Main Branch (Eq. 8 with the causal rule of Eq. 1) as a
// KV-outer block-sparse attention on tcgen05, in three steps per query chunk:
//
//   1. inverse index: for every (group r, block b) the list of selection slots
//      (query i, slot s) that chose b -- count, exclusive scan, scatter, each
//      CTA counting its range of slots in a shared-memory histogram of the
//      keys.  The scan also cuts each list into tiles of Tq queries (Tq *
//      rows-per-query = 128 MMA rows), so hot blocks are split over many CTAs
//      with every output slot fixed in advance: no atomics on the outputs.
//   2. phase 1: one tile = one KV block (K_b, V_b by TMA) and the gathered
//      query rows that selected it (one TMA box per query: its group's heads).
//      S = Q K_b^T (UMMA, fp32 in TMEM) -> causal mask (only rows whose own
//      block is b) -> softmax in registers (one row per thread, exp2) -> P
//      (bf16) to shared memory -> O = P V_b (UMMA) -> O / l written as an fp16
//      partial with its natural-log LSE into the row's slot.
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

#include <type_traits>

#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 320;
// Largest per-CTA key histogram of the inverse index (H_kv * B keys).
constexpr size_t kMaxHistBytes = 192 * 1024;
constexpr int kRowsPerTile = 128;
// Queries per chunk: bounds the partial-output workspace.  Chunks are kept
// large so that every (group, block) list holds many queries per chunk: K/V
// blocks are then reused over long runs of tiles (small chunks would keep the
// gathered Q in L2 but re-read K/V for nearly every tile at 1M tokens).
constexpr int kMaxChunk = 1 << 17;

// Rows per query inside an MMA tile: the group's G heads, or 8 heads (one
// 128-byte swizzle atom) when G < 8 (the extra heads are computed and dropped).
inline int rows_per_query(int G) { return G >= 8 ? G : 8; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct ChunkBufs {
  int32_t* counts;    // [nkeys]
  int32_t* offsets;   // [nkeys + 1]
  int32_t* tile_off;  // [nkeys + 1]
  int32_t* cursor;    // [nkeys]
  int32_t* n_tiles;   // [1]
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
  c.counts = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nkeys));
  c.cursor = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * nkeys));
  c.offsets = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (nkeys + 1)));
  c.tile_off = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * (nkeys + 1)));
  c.n_tiles = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * 4));
  c.entries = reinterpret_cast<uint32_t*>(take(sizeof(uint32_t) * slots));
  c.part_lse = reinterpret_cast<float*>(take(sizeof(float) * slots * G));
  c.part_o = reinterpret_cast<__half*>(take(sizeof(__half) * slots * G * d_h));
  *total = off;
  return c;
}

int64_t chunk_len(int64_t N, int B_k) {
  int64_t c = N < kMaxChunk ? N : kMaxChunk;
  return (c + B_k - 1) / B_k * B_k;
}

// ------------------------------------------------------------------ step 1 --
struct InvParams {
  const int32_t* idx;
  int64_t q0, nq;  // chunk [q0, q0 + nq)
  int H_kv, B_k, kk;
  int64_t B;
  int Tq;
  ChunkBufs c;
  DevStatus* status;
};

// The key (group r, block b) of entry e of the chunk, or -1 when the entry
// selects nothing (-1 padding, or a block after the query's own).  Entry e is
// (query, group, slot) in the layout of I, so e is also the entry's output
// slot id and I is read contiguously.
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
  return (b >= 0 && b <= i / p.B_k) ? r * static_cast<int>(p.B) + b : -1;
}

// Inverse index with a per-CTA histogram of every key in shared memory.  A
// CTA owns a contiguous range of entries (a range of queries).  Counting: the
// CTA counts its entries per key in shared memory and adds each non-zero
// count to the global one with a single atomic.  Scattering: the CTA counts
// again, reserves each key's range of the key's list with one atomic on the
// key's cursor, and places every entry at a shared-memory atomic's position
// inside that range.
template <bool SCATTER>
__global__ void __launch_bounds__(512) inv_index_smem_kernel(const InvParams p) {
  extern __shared__ int32_t hist[];  // [H_kv * B]
  const int nkeys = static_cast<int>(p.H_kv * p.B);
  const int64_t total = p.nq * p.H_kv * p.kk;
  const int64_t per = (total + gridDim.x - 1) / gridDim.x;
  const int64_t e0 = static_cast<int64_t>(blockIdx.x) * per;
  const int64_t e1 = e0 + per < total ? e0 + per : total;
  for (int j = threadIdx.x; j < nkeys; j += blockDim.x) hist[j] = 0;
  __syncthreads();
  for (int64_t e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
    const int key = inv_key(p, e, !SCATTER);
    if (key >= 0) atomicAdd(&hist[key], 1);
  }
  __syncthreads();
  if constexpr (!SCATTER) {
    for (int j = threadIdx.x; j < nkeys; j += blockDim.x) {
      const int n = hist[j];
      if (n > 0) atomicAdd(&p.c.counts[j], n);
    }
  } else {
    for (int j = threadIdx.x; j < nkeys; j += blockDim.x) {
      const int n = hist[j];
      if (n > 0) hist[j] = atomicAdd(&p.c.cursor[j], n);
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
    int key = -1;
    uint32_t slot = 0;
    if (t < total) {
      const int s = static_cast<int>(t / (p.nq * p.H_kv));
      const int64_t rem = t % (p.nq * p.H_kv);
      const int r = static_cast<int>(rem / p.nq);
      const int64_t il = rem % p.nq;
      const int64_t i = p.q0 + il;
      const int32_t b = p.idx[(i * p.H_kv + r) * p.kk + s];
      const int64_t b_i = i / p.B_k;
      if (b < -1 || b >= p.B) {
        if (!SCATTER) report(p.status, DEV_ERR_BAD_INDEX, 40, static_cast<int>(i), b);
      } else if (b >= 0 && b <= b_i) {
        key = r * static_cast<int>(p.B) + b;
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

// Single CTA: exclusive scans of the counts and of the per-key tile counts.
__global__ void __launch_bounds__(1024) inv_scan_kernel(const InvParams p) {
  __shared__ int32_t warp_sum[2][32];
  const int64_t nkeys = p.H_kv * p.B;
  const int per = static_cast<int>((nkeys + blockDim.x - 1) / blockDim.x);
  const int64_t beg = static_cast<int64_t>(threadIdx.x) * per;
  int32_t s_cnt = 0, s_til = 0;
  for (int j = 0; j < per; ++j) {
    const int64_t e = beg + j;
    if (e < nkeys) {
      const int32_t c = p.c.counts[e];
      s_cnt += c;
      s_til += (c + p.Tq - 1) / p.Tq;
    }
  }
  // block-wide exclusive scan of (s_cnt, s_til)
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int32_t a = s_cnt, b = s_til;
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t ya = __shfl_up_sync(0xFFFFFFFFu, a, o);
    const int32_t yb = __shfl_up_sync(0xFFFFFFFFu, b, o);
    if (lane >= o) {
      a += ya;
      b += yb;
    }
  }
  if (lane == 31) {
    warp_sum[0][w] = a;
    warp_sum[1][w] = b;
  }
  __syncthreads();
  if (w == 0) {
    int32_t x = lane < static_cast<int>(blockDim.x >> 5) ? warp_sum[0][lane] : 0;
    int32_t y = lane < static_cast<int>(blockDim.x >> 5) ? warp_sum[1][lane] : 0;
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t yx = __shfl_up_sync(0xFFFFFFFFu, x, o);
      const int32_t yy = __shfl_up_sync(0xFFFFFFFFu, y, o);
      if (lane >= o) {
        x += yx;
        y += yy;
      }
    }
    warp_sum[0][lane] = x;
    warp_sum[1][lane] = y;
  }
  __syncthreads();
  int32_t run_cnt = a - s_cnt + (w > 0 ? warp_sum[0][w - 1] : 0);
  int32_t run_til = b - s_til + (w > 0 ? warp_sum[1][w - 1] : 0);
  for (int j = 0; j < per; ++j) {
    const int64_t e = beg + j;
    if (e < nkeys) {
      const int32_t c = p.c.counts[e];
      p.c.offsets[e] = run_cnt;
      p.c.cursor[e] = run_cnt;
      p.c.tile_off[e] = run_til;
      run_cnt += c;
      run_til += (c + p.Tq - 1) / p.Tq;
    }
  }
  if (threadIdx.x == blockDim.x - 1) {
    p.c.offsets[nkeys] = run_cnt;
    p.c.tile_off[nkeys] = run_til;
    p.c.n_tiles[0] = run_til;
  }
}

// The inverse index's launch shape: a shared-memory histogram of every key per
// CTA when it fits (up to 4 CTAs per SM), else the global-atomic kernels.
cudaError_t inv_setup(int64_t nkeys, int sms, size_t* hist_bytes, int* hist_grid) {
  *hist_bytes = sizeof(int32_t) * static_cast<size_t>(nkeys);
  *hist_grid = sms;
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
  *hist_grid = sms * static_cast<int>(per_sm < 1 ? 1 : (per_sm > 4 ? 4 : per_sm));
  return cudaSuccess;
}

// Count -> scan -> scatter of one chunk's inverse index (counts zeroed before).
void launch_inv_index(const InvParams& ip, size_t hist_bytes, int hist_grid, int sms,
                      cudaStream_t stream) {
  const int64_t total = ip.nq * ip.H_kv * ip.kk;
  if (hist_bytes <= kMaxHistBytes) {
    prof_begin("inv_count", stream);
    inv_index_smem_kernel<false><<<hist_grid, 512, hist_bytes, stream>>>(ip);
    prof_end(stream);
    prof_begin("inv_scan", stream);
    inv_scan_kernel<<<1, 1024, 0, stream>>>(ip);
    prof_end(stream);
    prof_begin("inv_scatter", stream);
    inv_index_smem_kernel<true><<<hist_grid, 512, hist_bytes, stream>>>(ip);
    prof_end(stream);
  } else {
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > sms * 16) blocks = sms * 16;
    prof_begin("inv_count", stream);
    inv_index_kernel<false><<<blocks, 256, 0, stream>>>(ip);
    prof_end(stream);
    prof_begin("inv_scan", stream);
    inv_scan_kernel<<<1, 1024, 0, stream>>>(ip);
    prof_end(stream);
    prof_begin("inv_scatter", stream);
    inv_index_kernel<true><<<blocks, 256, 0, stream>>>(ip);
    prof_end(stream);
  }
}

// ------------------------------------------------------------------ step 2 --
struct P1Params {
  int64_t q0;
  int q4d;  // 1: one 4-D TMA box per gathered query ([d-chunk][head] rows, 8 heads)
  int H_q, H_kv, B_k, kk, G, R, Tq;
  int64_t nkeys;
  float scale_log2;  // softmax scale * log2(e)
  float scale;
  ChunkBufs c;
  DevStatus* status;
};

template <int D_H, int B_K>
struct P1Shape {
  static constexpr int QS = 5;   // Q/P ring depth
  static constexpr int NKV = 1;  // K/V slots (the ring and two slots do not both fit)
  static constexpr int QP_BYTES = kRowsPerTile * (D_H > B_K ? D_H : B_K) * 2;  // Q, later P
  static constexpr int K_BYTES = B_K * D_H * 2;
  static constexpr int V_BYTES = B_K * D_H * 2;
  static constexpr int DCH = D_H / 64;  // 128-byte chunks along d
  static constexpr int PCH = B_K / 64;  // 128-byte chunks along keys (P)
  static constexpr uint32_t TM_S = 0, TM_O = 128;  // column offsets inside a TMEM stage
};

constexpr int kMaxTq = 16;  // queries per tile (128 rows / at least 8 rows per query)

struct TileInfo {
  int r, b, len, gen;  // group, block, queries in the tile, K/V generation
  uint32_t slot[kMaxTq];
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
// block) key come in long runs there, so the K/V block sits in one shared
// slot for the whole run (reloaded only when the key changes) while the
// gathered query rows stream through a 5-deep ring.  TMEM holds two tiles
// (S and O, 128 + 128 columns each); two softmax/epilogue groups of four
// warps take alternate tiles.
//   warp 0      producer (all lanes: lane q issues query q's TMA box)
//   warp 1      MMA issuer (lane 0) and TMEM owner
//   warps 2..9  softmax + epilogue, group (w-2)/4
template <int D_H, int B_K>
__global__ void __launch_bounds__(kThreads, 1)
    attn_phase1_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const P1Params p) {
  using SH = P1Shape<D_H, B_K>;
  constexpr int QS = SH::QS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  // K/V slot j: K at sKV + j * (K_BYTES + V_BYTES), V right after it
  uint8_t* sKV = smem + QS * SH::QP_BYTES;
  TileInfo* info = reinterpret_cast<TileInfo*>(sKV + SH::NKV * (SH::K_BYTES + SH::V_BYTES));
  uint64_t* bars = reinterpret_cast<uint64_t*>(info + QS);
  uint64_t* q_full = bars;             // [QS] gathered Q landed
  uint64_t* q_empty = q_full + QS;     // [QS] stage free: partials of its tile copied out
  uint64_t* kv_full = q_empty + QS;    // [NKV] K/V block landed
  uint64_t* kv_empty = kv_full + SH::NKV;  // [NKV] last tile of a K/V run finished O = P V
  uint64_t* s_full = kv_empty + SH::NKV;   // [2] S in TMEM
  uint64_t* p_full = s_full + 2;       // [2] P in smem (S read)
  uint64_t* o_full = p_full + 2;       // [2] O in TMEM
  uint64_t* o_empty = o_full + 2;      // [2] O read
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 4);  // the tile's 4 epilogue warps, after their bulk stores
    }
    for (int j = 0; j < SH::NKV; ++j) {
      mbar_init(&kv_full[j], 1);
      mbar_init(&kv_empty[j], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
      mbar_init(&o_full[s], 1);
      mbar_init(&o_empty[s], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_tiles = p.c.n_tiles[0];
  // contiguous tile range of this CTA (tiles are equal-sized units of work)
  const int t_beg = static_cast<int>(static_cast<int64_t>(n_tiles) * blockIdx.x / gridDim.x);
  const int t_end = static_cast<int>(static_cast<int64_t>(n_tiles) * (blockIdx.x + 1) / gridDim.x);
  const int my_tiles = t_end - t_beg;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
    }
    const int nb = static_cast<int>(p.nkeys / p.H_kv);
    const int per_q = p.H_kv * p.kk;
    // tile cursor: key, its first tile, its entry range
    int key = 0, kt0 = 0, kend = 0, koff = 0, kcnt = 0;
    auto seek = [&](int t) {
      while (kend <= t) {
        ++key;
        kt0 = p.c.tile_off[key];
        kend = p.c.tile_off[key + 1];
      }
      koff = p.c.offsets[key];
      kcnt = p.c.offsets[key + 1] - koff;
    };
    uint32_t next_slot = 0;
    int next_len = 0;
    if (my_tiles > 0) {
      key = find_key(p.c.tile_off, p.nkeys, t_beg);
      kt0 = p.c.tile_off[key];
      kend = p.c.tile_off[key + 1];
      koff = p.c.offsets[key];
      kcnt = p.c.offsets[key + 1] - koff;
      const int lt = t_beg - kt0;
      next_len = min(p.Tq, kcnt - lt * p.Tq);
      if (lane < next_len) next_slot = p.c.entries[koff + lt * p.Tq + lane];
    }
    int kv_key = -1, kvgen = 0;
    for (int n = 0; n < my_tiles; ++n) {
      const int t = t_beg + n;
      const int cur_key = key, len = next_len;
      const uint32_t myslot = next_slot;
      const int r = cur_key / nb, b = cur_key - r * nb;
      // fetch the next tile's slots now; their latency hides behind the waits
      if (n + 1 < my_tiles) {
        if (t + 1 >= kend) seek(t + 1);
        const int lt = t + 1 - kt0;
        next_len = min(p.Tq, kcnt - lt * p.Tq);
        next_slot = lane < next_len ? p.c.entries[koff + lt * p.Tq + lane] : 0u;
      }
      const bool new_kv = cur_key != kv_key;
      const int gen = new_kv ? kvgen : kvgen - 1;
      // Q of this tile first (the MMA warp needs it to see a K/V switch)
      const int qs = n % QS;
      if (!mbar_wait(&q_empty[qs], ((n / QS) & 1) ^ 1, abort_flag, p.status, 50)) break;
      TileInfo& ti = info[qs];
      if (lane < len) ti.slot[lane] = myslot;
      if (lane == 0) {
        ti.r = r;
        ti.b = b;
        ti.len = len;
        ti.gen = gen;
        mbar_arrive_expect_tx(&q_full[qs], len * p.R * D_H * 2);
      }
      __syncwarp();
      const int h0 = p.G >= 8 ? r * p.G : (r * p.G / 8) * 8;
      if (lane < len) {
        const int i = static_cast<int>(p.q0 + myslot / per_q);
        uint8_t* sQ = smem + qs * SH::QP_BYTES;
        if (p.q4d) {
          // query-major: [query][d-chunk][8 heads x 128 B]
          tma_load_4d(sQ + lane * 8 * D_H * 2, &tm_q, &q_full[qs], 0, h0, 0, i);
        } else {
          // chunk-major: [d-chunk][query rows x 128 B]
#pragma unroll
          for (int c = 0; c < SH::DCH; ++c)
            tma_load_3d(sQ + c * kRowsPerTile * 128 + lane * p.R * 128, &tm_q, &q_full[qs],
                        c * 64, h0, i);
        }
      }
      if (new_kv) {
        // generation g lives in slot g % NKV; the slot is free once every tile
        // of generation g - NKV finished O = P V
        const int slot = kvgen % SH::NKV;
        if (kvgen >= SH::NKV &&
            !mbar_wait(&kv_empty[slot], ((kvgen / SH::NKV) - 1) & 1, abort_flag, p.status, 51))
          break;
        uint8_t* sK = sKV + slot * (SH::K_BYTES + SH::V_BYTES);
        uint8_t* sV = sK + SH::K_BYTES;
        if (lane == 0) mbar_arrive_expect_tx(&kv_full[slot], SH::K_BYTES + SH::V_BYTES);
        __syncwarp();
        if (lane < SH::DCH) {
          tma_load_3d(sK + lane * B_K * 128, &tm_k, &kv_full[slot], lane * 64, r, b * B_K);
          tma_load_3d(sV + lane * B_K * 128, &tm_v, &kv_full[slot], lane * 64, r, b * B_K);
        }
        kv_key = cur_key;
        ++kvgen;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    // S of tile n+1 is issued before waiting for the softmax of tile n, so the
    // tensor core works while P is built.  After O(n) of a run's last tile the
    // run's K/V slot is released; with a single slot the next run's K/V can
    // only land after that, so at a switch O(n) goes first.
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, B_K, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D_H, 0, 1);
      int gen_have = -1;
      auto wait_q = [&](int n, int* gen) -> bool {
        const int qs = n % QS;
        if (!mbar_wait(&q_full[qs], (n / QS) & 1, abort_flag, p.status, 60)) return false;
        *gen = info[qs].gen;
        return true;
      };
      auto issue_s = [&](int n, int gen) -> bool {
        if (gen != gen_have) {
          if (!mbar_wait(&kv_full[gen % SH::NKV], (gen / SH::NKV) & 1, abort_flag, p.status, 63))
            return false;
          gen_have = gen;
        }
        tc_fence_after();
        const uint32_t q_base = smem_u32(smem + (n % QS) * SH::QP_BYTES);
        const uint32_t k_base = smem_u32(sKV + (gen % SH::NKV) * (SH::K_BYTES + SH::V_BYTES));
        const uint32_t tS = tmem_base + (n & 1) * 256 + SH::TM_S;
        // 8-row groups: consecutive queries (query-major) or consecutive rows
        const uint32_t q_sbo = p.q4d ? 8 * D_H * 2 : 1024;
        const uint32_t q_cstep = p.q4d ? 8 * 128 : kRowsPerTile * 128;
#pragma unroll
        for (int c = 0; c < SH::DCH; ++c)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint64_t ad = umma_desc(q_base + c * q_cstep + s * 32, 16, q_sbo, SW_128B);
            const uint64_t bd = umma_desc(k_base + c * B_K * 128 + s * 32, 16, 1024, SW_128B);
            umma_bf16(tS, ad, bd, idesc_s, (c | s) != 0);
          }
        umma_commit(&s_full[n & 1]);
        return true;
      };
      int gcur = 0;
      bool ok = my_tiles == 0 || (wait_q(0, &gcur) && issue_s(0, gcur));
      for (int n = 0; ok && n < my_tiles; ++n) {
        const int st = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        const bool has_next = n + 1 < my_tiles;
        // S of tile n+1 goes before O(n) only if its gathered rows have
        // already landed: O(n) must never wait behind the next gather.  (S of
        // tile n+1 reuses the TMEM stage of tile n-1, whose P was waited for in
        // the previous iteration.)
        int gnext = gcur;
        bool s_done = false;
        if (has_next && mbar_try_wait(&q_full[(n + 1) % QS], ((n + 1) / QS) & 1)) {
          gnext = info[(n + 1) % QS].gen;
          if (SH::NKV > 1 || gnext == gcur) {
            if (!issue_s(n + 1, gnext)) break;
            s_done = true;
          }
        }
        if (!mbar_wait(&p_full[st], ph, abort_flag, p.status, 61)) break;
        if (!mbar_wait(&o_empty[st], ph ^ 1, abort_flag, p.status, 62)) break;
        tc_fence_after();
        const uint32_t q_base = smem_u32(smem + (n % QS) * SH::QP_BYTES);
        const uint32_t v_base =
            smem_u32(sKV + (gcur % SH::NKV) * (SH::K_BYTES + SH::V_BYTES) + SH::K_BYTES);
        const uint32_t tO = tmem_base + st * 256 + SH::TM_O;
#pragma unroll
        for (int c = 0; c < SH::PCH; ++c)
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            // P: K-major (keys contiguous), chunk c = keys [64c, 64c+64)
            const uint64_t ad =
                umma_desc(q_base + c * kRowsPerTile * 128 + s * 32, 16, 1024, SW_128B);
            // V: MN-major (d contiguous); 16 keys = two 8-key groups = 2048 B
            const uint64_t bd = umma_desc(v_base + (c * 4 + s) * 2048, B_K * 128, 1024, SW_128B);
            umma_bf16(tO, ad, bd, idesc_o, (c | s) != 0);
          }
        umma_commit(&o_full[st]);
        if (has_next && !s_done) {
          if (!wait_q(n + 1, &gnext)) break;
          // a run's last tile releases its K/V slot once O(n) has finished
          if (gnext != gcur) umma_commit(&kv_empty[gcur % SH::NKV]);
          if (!issue_s(n + 1, gnext)) break;
        } else if (has_next && gnext != gcur) {
          umma_commit(&kv_empty[gcur % SH::NKV]);
        }
        gcur = gnext;
      }
    }
  } else {
    // ------------------------------------------ softmax + epilogue groups --
    const int grp = (warp - 2) >> 2;  // handles tiles n with n % 2 == grp
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int q_local = row / p.R;
    const int hrow = row - q_local * p.R;
    const int per_q = p.H_kv * p.kk;
    for (int n = grp; n < my_tiles; n += 2) {
      const int st = grp;
      const uint32_t ph = (n >> 1) & 1;
      const int qs = n % QS;
      uint8_t* sP = smem + qs * SH::QP_BYTES;
      const uint32_t tS = tmem_base + st * 256 + SH::TM_S + (static_cast<uint32_t>(quarter * 32) << 16);
      const uint32_t tO = tmem_base + st * 256 + SH::TM_O + (static_cast<uint32_t>(quarter * 32) << 16);
      if (!mbar_wait(&s_full[st], ph, abort_flag, p.status, 70)) break;
      // q_full[qs] cannot advance before this tile's O MMA, so this returns at
      // once; it orders the producer's TileInfo writes before the reads below
      if (!mbar_wait(&q_full[qs], (n / QS) & 1, abort_flag, p.status, 72)) break;
      tc_fence_after();
      const int ti_r = info[qs].r, ti_b = info[qs].b, ti_len = info[qs].len;
      const bool live = q_local < ti_len;
      const uint32_t slot = live ? info[qs].slot[q_local] : 0u;
      const int64_t i = p.q0 + slot / per_q;
      // ---- softmax over the block's keys (exp2 with the scale folded in)
      float sv[B_K];
      {
        uint32_t r32[B_K / 32][32];
#pragma unroll
        for (int c = 0; c < B_K / 32; ++c) tmem_ld32(tS + c * 32, r32[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < B_K / 32; ++c)
#pragma unroll
          for (int j = 0; j < 32; ++j) sv[c * 32 + j] = __uint_as_float(r32[c][j]);
      }
      const int64_t j0 = static_cast<int64_t>(ti_b) * B_K;
      if (j0 + B_K - 1 > i) {  // the query's own block: causal rule j <= i
#pragma unroll
        for (int j = 0; j < B_K; ++j)
          if (j0 + j > i) sv[j] = -INFINITY;
      }
      float mx = sv[0];
#pragma unroll
      for (int j = 1; j + 1 < B_K; j += 2) mx = fmax3(mx, sv[j], sv[j + 1]);
      mx = fmaxf(mx, sv[B_K - 1]);
      const float mscaled = mx * p.scale_log2;
      float l = 0.0f;
#pragma unroll
      for (int j = 0; j < B_K; ++j) {
        const float e = exp2f(fmaf(sv[j], p.scale_log2, -mscaled));
        sv[j] = e;
        l += e;
      }
      // P (bf16) over the stage's Q rows (consumed by S), K-major 128B-swizzled
#pragma unroll
      for (int c = 0; c < B_K / 8; ++c) {
        uint4 w;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(sv[c * 8 + 0], sv[c * 8 + 1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(sv[c * 8 + 2], sv[c * 8 + 3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(sv[c * 8 + 4], sv[c * 8 + 5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(sv[c * 8 + 6], sv[c * 8 + 7]);
        w.x = *reinterpret_cast<uint32_t*>(&h0);
        w.y = *reinterpret_cast<uint32_t*>(&h1);
        w.z = *reinterpret_cast<uint32_t*>(&h2);
        w.w = *reinterpret_cast<uint32_t*>(&h3);
        const int kc = c >> 3, j16 = c & 7;
        uint8_t* dst = sP + kc * kRowsPerTile * 128 + row * 128 + ((j16 ^ (row & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = w;
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
      // ---- O = P V; write O / l as an fp16 partial and lse into the slot
      if (!mbar_wait(&o_full[st], ph, abort_flag, p.status, 71)) break;
      tc_fence_after();
      const int goff = p.G >= 8 ? 0 : (ti_r * p.G) % 8;  // group's first head in the box
      const bool useful = live && hrow >= goff && hrow < goff + p.G;
      const int g = hrow - goff;
      // partial layout [slot][d/8][g][8].  The tile's partials are staged in its
      // Q/P buffer (P is dead once O = P V completed) in exactly that layout,
      // so each query's G x d_h block is one contiguous bulk copy to HBM.
      const int qbytes = p.G * D_H * 2;  // one query's partial block
      uint8_t* stage = sP + q_local * qbytes;
      const float inv_l = 1.0f / l;
      uint32_t ro[D_H / 32][32];
#pragma unroll
      for (int c = 0; c < D_H / 32; ++c) tmem_ld32(tO + c * 32, ro[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty[st]);
      if (useful) {
#pragma unroll
        for (int c = 0; c < D_H / 32; ++c)
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 w;
            __half2 a0 = __floats2half2_rn(__uint_as_float(ro[c][j + 0]) * inv_l, __uint_as_float(ro[c][j + 1]) * inv_l);
            __half2 a1 = __floats2half2_rn(__uint_as_float(ro[c][j + 2]) * inv_l, __uint_as_float(ro[c][j + 3]) * inv_l);
            __half2 a2 = __floats2half2_rn(__uint_as_float(ro[c][j + 4]) * inv_l, __uint_as_float(ro[c][j + 5]) * inv_l);
            __half2 a3 = __floats2half2_rn(__uint_as_float(ro[c][j + 6]) * inv_l, __uint_as_float(ro[c][j + 7]) * inv_l);
            w.x = *reinterpret_cast<uint32_t*>(&a0);
            w.y = *reinterpret_cast<uint32_t*>(&a1);
            w.z = *reinterpret_cast<uint32_t*>(&a2);
            w.w = *reinterpret_cast<uint32_t*>(&a3);
            *reinterpret_cast<uint4*>(stage + (((c * 32 + j) >> 3) * p.G + g) * 16) = w;
          }
      }
      fence_async_smem();
      __syncwarp();
      // one lane per query (its first useful head) copies the query's block
      if (useful && g == 0) {
        bulk_store(p.c.part_o + static_cast<int64_t>(slot) * p.G * D_H, stage, qbytes);
        bulk_commit();
        bulk_wait_read_all();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[qs]);
      if (useful) {
        p.c.part_lse[static_cast<int64_t>(slot) * p.G + g] = mx * p.scale + logf(l);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
  const int64_t b_i = i / p.B_k;
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
  const int64_t b_i = i / p.B_k;
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
  return 1024 + SH::QS * SH::QP_BYTES + SH::NKV * (SH::K_BYTES + SH::V_BYTES) +
         SH::QS * sizeof(TileInfo) + (2 * SH::QS + 2 * SH::NKV + 8) * 8 + 16;
}

template <int D_H, int B_K>
cudaError_t launch_typed(const AttnLaunch& a, cudaStream_t stream) {
  const int G = a.H_q / a.H_kv;
  const int R = rows_per_query(G);
  const int Tq = kRowsPerTile / R;
  const int64_t B = (a.N + a.B_k - 1) / a.B_k;
  const int64_t nkeys = a.H_kv * B;
  const int64_t Nc = chunk_len(a.N, a.B_k);
  size_t need = 0;
  ChunkBufs c = carve(a.ws, Nc, a.H_q, a.H_kv, a.d_h, a.kk, nkeys, &need);
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
  e = inv_setup(nkeys, sms, &hist_bytes, &hist_grid);
  if (e != cudaSuccess) return e;

  for (int64_t q0 = 0; q0 < a.N; q0 += Nc) {
    const int64_t nq = (a.N - q0) < Nc ? (a.N - q0) : Nc;
    e = cudaMemsetAsync(c.counts, 0, sizeof(int32_t) * nkeys, stream);
    if (e != cudaSuccess) return e;
    InvParams ip;
    ip.idx = a.idx;
    ip.q0 = q0;
    ip.nq = nq;
    ip.H_kv = a.H_kv;
    ip.B_k = a.B_k;
    ip.kk = a.kk;
    ip.B = B;
    ip.Tq = Tq;
    ip.c = c;
    ip.status = a.status;
    launch_inv_index(ip, hist_bytes, hist_grid, sms, stream);

    P1Params pp;
    pp.q0 = q0;
    pp.q4d = q4d;
    pp.H_q = a.H_q;
    pp.H_kv = a.H_kv;
    pp.B_k = a.B_k;
    pp.kk = a.kk;
    pp.G = G;
    pp.R = R;
    pp.Tq = Tq;
    pp.nkeys = nkeys;
    pp.scale = a.scale;
    pp.scale_log2 = a.scale * 1.4426950408889634f;
    pp.c = c;
    pp.status = a.status;
    prof_begin("attn_phase1", stream);
    attn_phase1_kernel<D_H, B_K><<<sms, kThreads, smem, stream>>>(tq, tk, tv, pp);
    prof_end(stream);

    MergeParams mp;
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
    InvParams ip;
    ip.idx = a.idx;
    ip.q0 = q0;
    ip.nq = nq;
    ip.H_kv = a.H_kv;
    ip.B_k = B_K;
    ip.kk = a.kk;
    ip.B = B;
    ip.Tq = kLseTile;
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

size_t attn_workspace_bytes(int64_t N, int H_q, int H_kv, int d_h, int B_k, int kk) {
  const int64_t B = (N + B_k - 1) / B_k;
  size_t total = 0;
  carve(nullptr, chunk_len(N, B_k), H_q, H_kv, d_h, kk, H_kv * B, &total);
  return total;
}

cudaError_t launch_sparse_attn(const AttnLaunch& a, cudaStream_t s) {
  if (a.d_h == 128 && a.B_k == 128) return launch_typed<128, 128>(a, s);
  if (a.d_h == 128 && a.B_k == 64) return launch_typed<128, 64>(a, s);
  if (a.d_h == 64 && a.B_k == 128) return launch_typed<64, 128>(a, s);
  if (a.d_h == 64 && a.B_k == 64) return launch_typed<64, 64>(a, s);
  return cudaErrorInvalidValue;
}

}  // namespace msa
