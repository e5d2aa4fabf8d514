// varlen.cu -- tables for several sequences packed along the token axis.
//
// A batch of prefill sequences is one tensor per input with the sequences
// one after another (cu_seqlens: sequence s holds tokens cu[s] .. cu[s+1]-1,
// any lengths, no padding).  Everything the method computes stays inside a
// sequence (Eq. 1 and 6-8 of the xllm-io paper review, "核心公式", read per
// sequence): block b of sequence s is its tokens cu[s] + b*B_k ..., a query's
// candidate blocks are the earlier blocks of its own sequence and its local
// block is (i - cu[s]) / B_k.  The kernels see this through three tables:
//   qinfo[i]   = {cu[s], blk_base[s]} for the sequence s of token i, where
//                blk_base numbers the blocks of all sequences globally (the
//                inverse index's keys);
//   blk_row[g] = the first token of global block g;
//   tiles[u]   = the index kernel's M-tiles (128 Q_idx rows of one sequence),
//                longest candidate range first: {first Q_idx row, cu[s],
//                local block of the tile's queries, valid rows}.
#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kTileRows = 128;  // Q_idx rows of the index kernel's M-tile

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Counts {
  int64_t B_tot = 0;
  int64_t n_tiles = 0;
};

Counts count(const int64_t* cu, int n, int B_k, int H_kv) {
  Counts c;
  for (int s = 0; s < n; ++s) {
    const int64_t len = cu[s + 1] - cu[s];
    c.B_tot += (len + B_k - 1) / B_k;
    c.n_tiles += (len * H_kv + kTileRows - 1) / kTileRows;
  }
  return c;
}

// Thread t < N: token t's sequence (the last s with cu[s] <= t, which skips
// empty sequences); thread t < B_tot: global block t's first token.
__global__ void varlen_fill_kernel(const int2* seq, int n, int64_t N, int64_t B_tot, int B_k,
                                   int2* qinfo, int32_t* blk_row) {
  const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (t < N) {
    int lo = 0, hi = n;  // seq[lo].x <= t < seq[hi].x
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (seq[mid].x <= t) lo = mid;
      else hi = mid;
    }
    qinfo[t] = seq[lo];
  }
  if (t < B_tot) {
    int lo = 0, hi = n;  // seq[lo].y <= t < seq[hi].y
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (seq[mid].y <= t) lo = mid;
      else hi = mid;
    }
    blk_row[t] = seq[lo].x + static_cast<int32_t>(t - seq[lo].y) * B_k;
  }
}

}  // namespace

size_t varlen_table_bytes(const int64_t* cu, int n, int B_k, int H_kv, bool tiles) {
  const Counts c = count(cu, n, B_k, H_kv);
  const int64_t N = cu[n];
  return align256(sizeof(int2) * (n + 1)) + align256(sizeof(int2) * N) +
         align256(sizeof(int32_t) * (c.B_tot > 0 ? c.B_tot : 1)) +
         (tiles ? align256(sizeof(int4) * (c.n_tiles > 0 ? c.n_tiles : 1)) : 0);
}

cudaError_t build_varlen_tables(const int64_t* cu, int n, int B_k, int H_kv, bool tiles,
                                void* dst, VarlenTables* out, cudaStream_t s) {
  const Counts c = count(cu, n, B_k, H_kv);
  const int64_t N = cu[n];
  uint8_t* p = static_cast<uint8_t*>(dst);
  int2* d_seq = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * (n + 1));
  int2* d_qinfo = reinterpret_cast<int2*>(p);
  p += align256(sizeof(int2) * N);
  int32_t* d_blk_row = reinterpret_cast<int32_t*>(p);
  p += align256(sizeof(int32_t) * (c.B_tot > 0 ? c.B_tot : 1));
  int4* d_tiles = tiles ? reinterpret_cast<int4*>(p) : nullptr;

  // per sequence {first token, first global block}, with the end as entry n
  std::vector<int2> seq(n + 1);
  int64_t base = 0;
  for (int i = 0; i <= n; ++i) {
    seq[i] = make_int2(static_cast<int>(cu[i]), static_cast<int>(base));
    if (i < n) base += (cu[i + 1] - cu[i] + B_k - 1) / B_k;
  }
  cudaError_t e = cudaMemcpyAsync(d_seq, seq.data(), sizeof(int2) * (n + 1),
                                  cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  if (tiles && c.n_tiles > 0) {
    std::vector<int4> list;
    list.reserve(static_cast<size_t>(c.n_tiles));
    for (int i = 0; i < n; ++i) {
      const int64_t rows = (cu[i + 1] - cu[i]) * H_kv;
      for (int64_t r0 = 0; r0 < rows; r0 += kTileRows) {
        const int local_block = static_cast<int>(r0 / H_kv / B_k);
        const int64_t left = rows - r0;
        list.push_back(make_int4(static_cast<int>(cu[i] * H_kv + r0), static_cast<int>(cu[i]),
                                 local_block, static_cast<int>(left < kTileRows ? left : kTileRows)));
      }
    }
    // longest candidate range first, so the last tiles of the persistent
    // grid are short ones
    std::stable_sort(list.begin(), list.end(),
                     [](const int4& a, const int4& b) { return a.z > b.z; });
    e = cudaMemcpyAsync(d_tiles, list.data(), sizeof(int4) * list.size(), cudaMemcpyHostToDevice,
                        s);
    if (e != cudaSuccess) return e;
  }
  const int64_t work = N > c.B_tot ? N : c.B_tot;
  if (work > 0) {
    varlen_fill_kernel<<<static_cast<unsigned>((work + 255) / 256), 256, 0, s>>>(
        d_seq, n, N, c.B_tot, B_k, d_qinfo, d_blk_row);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  out->qinfo = d_qinfo;
  out->blk_row = d_blk_row;
  out->tiles = d_tiles;
  out->n_tiles = static_cast<int>(c.n_tiles);
  out->B_tot = c.B_tot;
  return cudaSuccess;
}

int64_t varlen_blocks(const int64_t* cu, int n, int B_k) { return count(cu, n, B_k, 1).B_tot; }

}  // namespace msa
