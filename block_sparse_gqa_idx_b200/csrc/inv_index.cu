// inv_index.cu -- the inverse index of a query chunk's selection: for every
// (group r, block b) key the list of selection slots (query i, slot s) that
// chose b -- count, exclusive scan (multi-CTA), scatter, each CTA counting
// its range of slots in a shared-memory histogram of the keys.  The scan also
// cuts each list into tiles of Tq queries and writes each tile's (key, first
// entry, length, the key's end tile), so hot blocks are split over many CTAs
// with every output slot fixed in advance: no atomics on the outputs.
//
// Source: chlience notes 3 (the reverse index as an overhead of the method)
// and 5.4 (pre-scheduled tile chunking, slots assigned ahead).
#include "attn_common.cuh"

namespace msa {
namespace {

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

}  // namespace

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

}  // namespace msa
