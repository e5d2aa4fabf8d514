// index_topk.cu -- fused Index Branch kernel: Eq. 6 scores on tcgen05, causal
// block max-pool in registers, Eq. 7 Top-k with the local block forced.
//
// Source: xllm-io paper review, "核心公式" (Eq. 6-7) and "4.1 Index & TopK
// Kernel"; chlience notes 5.1.1 (local block takes one slot) and 5.4
// (exp-free selection: rank raw scores).
//
// Design (sm_100a):
//   * Rows of the MMA are (query, group) pairs: Q_idx is [N, H_kv, d_idx], so
//     128 consecutive rows of the [N*H_kv, d_idx] view are 128/H_kv queries x
//     all H_kv groups, and they all share the one index key head (Eq. 5).  A
//     work unit is one such 128-row M-tile; every 256-key K_idx tile streamed
//     by TMA feeds one 128x256xd_idx UMMA (A = Q_idx rows, B = K_idx rows,
//     both K-major, fp32 accumulators in TMEM).  At N = 256 an MMA step reads
//     96 bytes of shared-memory operands per clock at peak rate, against 128
//     (all of it) for two N = 128 MMAs, which measured about 20% slower.
//   * All queries of an M-tile live in one block c (128/H_kv divides B_k), so
//     the non-local candidates are exactly blocks 0..c-1: every key tile is
//     fully visible and needs no causal mask.  The local block is forced and
//     needs no score at all.
//   * Epilogue: one TMEM lane (= one row) per thread; two groups of four
//     warps read the two 128-column halves of a tile (at B_k = 128 the even
//     and the odd blocks).  tcgen05.ld pulls a row's 128 scores of the half,
//     a 3-input max tree pools them per block, and each group keeps its own
//     running Top-(k-1) of packed keys (score bits, inverted block index): a
//     sorted register list for k <= 16, else a min-heap in shared memory
//     whose root score is cached in a register, so a block costs one compare
//     unless it enters.  At the end of a unit group 1 hands its list to
//     group 0 through shared memory and group 0 merges the two and writes the
//     row.  The scale 1/sqrt(d_idx) is positive and is not applied: the order
//     of the raw dot products is the order of Eq. 6's scores.
//   * Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer (and TMEM
//     owner), warps 2..9 = epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).
//     TMEM holds 2 accumulator stages x 256 columns = 512 columns.
//   * Persistent grid of one CTA per SM; units are visited longest-first in a
//     snake order over CTAs to balance the causal triangle.
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_internal.h"

namespace msa {
namespace {

constexpr int kThreads = 320;
constexpr int kRows = 128;           // rows per M-tile (UMMA M)
constexpr int kKeys = 256;           // keys per K_idx tile (UMMA N)
constexpr int kHalf = 128;           // key columns of a tile read by one epilogue group
constexpr int kEpiThreads = 256;     // 2 groups x 128 rows
constexpr uint32_t kTmemCols = 512;  // 2 accumulator stages x 256 columns
constexpr int kMaxHeap = 31;         // k - 1 for the largest supported k

struct IndexParams {
  int64_t N;
  int H_kv, B_k, k;
  int n_mtiles;
  // several sequences packed along the token axis: one record per M-tile,
  // longest first, {first Q_idx row, first token of the tile's sequence,
  // local block of its queries, valid rows}; and per token {first token of
  // its sequence, first global block of its sequence}.  Both null for one
  // sequence.
  const int4* tiles;
  const int2* qinfo;
  int32_t* idx_out;
  float* score_out;  // [N, H_kv, k] or null: the selected blocks' Eq. 6 scores
  float scale;       // Eq. 6 scale applied to score_out
  DevStatus* status;
};

template <int D_IDX>
struct IndexShape {
  static constexpr int SWB = (D_IDX * 2 < 128) ? D_IDX * 2 : 128;  // swizzle span (bytes)
  static constexpr int CH = D_IDX * 2 / SWB;                       // K chunks
  static constexpr int CHE = SWB / 2;                              // elements per chunk
  static constexpr int KSTEPS = SWB / 32;                          // UMMA K=16 steps per chunk
  static constexpr uint32_t SWZ = (SWB == 128) ? SW_128B : SW_64B;
  static constexpr int SBO = 8 * SWB;                              // 8-row atom
  static constexpr int A_BYTES = kRows * D_IDX * 2;                // one M-tile
  static constexpr int B_BYTES = kKeys * D_IDX * 2;                // one key tile
  // key tiles in flight: what shared memory holds beside A and the per-row
  // Top-k keys (sized for the largest k)
  static constexpr int FIXED = 1024 + A_BYTES + kEpiThreads * kMaxHeap * 8 + 512;
  static constexpr int FIT = (227 * 1024 - FIXED) / B_BYTES;
  static constexpr int STAGES = FIT > 6 ? 6 : FIT;
  static_assert(STAGES >= 2, "two key tiles must fit");
};

__device__ __forceinline__ int unit_of(int round, int cta, int nctas) {
  return round * nctas + ((round & 1) ? (nctas - 1 - cta) : cta);
}

// Work unit u (longest first): the M-tile's first Q_idx row, the first key
// row of its sequence, the local block c of its queries (relative to the
// sequence) and its valid rows.  Its candidate blocks 0..c-1 of the sequence
// are keys key0 .. key0 + c*B_k - 1.
struct MTile {
  int64_t row0, key0;
  int c, nrows;
};
__device__ __forceinline__ MTile mtile_of(const IndexParams& p, int u) {
  MTile t;
  if (p.tiles != nullptr) {
    const int4 r = p.tiles[u];
    t.row0 = r.x;
    t.key0 = r.y;
    t.c = r.z;
    t.nrows = r.w;
  } else {
    const int m = p.n_mtiles - 1 - u;
    t.row0 = static_cast<int64_t>(m) * kRows;
    t.key0 = 0;
    t.c = static_cast<int>(t.row0 / p.H_kv / p.B_k);
    const int64_t left = p.N * p.H_kv - t.row0;
    t.nrows = left < kRows ? static_cast<int>(left) : kRows;
  }
  return t;
}
// 256-key tiles holding the candidate blocks 0..c-1 (0 when c = 0).
__device__ __forceinline__ int mtile_ntiles(const IndexParams& p, const MTile& t) {
  return static_cast<int>((static_cast<int64_t>(t.c) * p.B_k + kKeys - 1) / kKeys);
}

// Top-k keys: the score's order-preserving bits above the inverted block
// index, so a larger key is a higher score or, at equal scores, a lower
// block (Eq. 7 with ties to the lower index).  0 is an empty slot.
__device__ __forceinline__ uint32_t order_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ uint64_t pack_key(float score, int b) {
  return (static_cast<uint64_t>(order_bits(score)) << 32) |
         static_cast<uint64_t>(0xFFFFFFFFu - static_cast<uint32_t>(b));
}
__device__ __forceinline__ int key_block(uint64_t key) {
  return static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(key));
}
__device__ __forceinline__ float unorder_key(uint64_t key) {
  if (key == 0) return -INFINITY;  // empty slot
  const uint32_t o = static_cast<uint32_t>(key >> 32);
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7FFFFFFFu) : ~o);
}

// A work unit is one M-tile of 128 rows against 256-key K_idx tiles: one
// 128x256xd_idx UMMA per tile (the wide N halves the shared-memory operand
// bytes per FLOP against two 128-wide MMAs).  Epilogue group g reads the
// tile's columns [128g, 128g+128) -- at B_k = 128 the even or the odd blocks
// -- and keeps its own running Top-(k-1) of them; at the end of the unit
// group 1 hands its list to group 0 through shared memory and group 0 merges
// the two and writes the row.
// REG: the running list lives in registers (k <= 16, a branch-free sorted
// insertion network); otherwise in a shared-memory min-heap.
// 10 warps: three of them share one SM sub-partition's 16K registers, so the
// kernel lives within 168 registers per thread; one CTA per SM.
template <int D_IDX, bool REG>
__global__ void __launch_bounds__(kThreads, 1)
    index_topk_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const IndexParams p) {
  using S = IndexShape<D_IDX>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                                   // A_BYTES
  uint8_t* sB = sA + S::A_BYTES;                        // STAGES x B_BYTES
  // [HS][kEpiThreads] Top-k keys per (slot, group column): the running heap
  // (shared-memory path) and the hand-over to group 0 (both paths)
  uint64_t* keys = reinterpret_cast<uint64_t*>(sB + S::STAGES * S::B_BYTES);
  const int HS = p.k - 1;                               // non-local slots per row
  uint64_t* bars = keys + static_cast<size_t>(kEpiThreads) * (HS > 0 ? HS : 1);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* b_full = bars + 2;
  uint64_t* b_empty = b_full + S::STAGES;
  uint64_t* acc_full = b_empty + S::STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* xch_full = acc_empty + 2;   // group 1's list is in shared memory
  uint64_t* xch_empty = xch_full + 1;   // group 0 has read it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(xch_empty + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < S::STAGES; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 8);
    }
    mbar_init(xch_full, 4);
    mbar_init(xch_empty, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int nctas = gridDim.x;
  const int cta = blockIdx.x;

  if (warp == 0) {
    // ------------------------------------------------------- TMA producer --
    if (lane == 0) {
      uint32_t g = 0, ua = 0;
      for (int round = 0;; ++round) {
        const int u = unit_of(round, cta, nctas);
        if (u >= p.n_mtiles || *abort_flag) break;
        const MTile mt = mtile_of(p, u);  // longest first
        const int nt = mtile_ntiles(p, mt);
        if (nt == 0) continue;
        if (!mbar_wait(a_empty, (ua & 1) ^ 1, abort_flag, p.status, 10)) break;
        mbar_arrive_expect_tx(a_full, S::A_BYTES);
        for (int ch = 0; ch < S::CH; ++ch)
          tma_load_2d(sA + ch * kRows * S::SWB, &tm_q, a_full, ch * S::CHE,
                      static_cast<int>(mt.row0));
        ++ua;
        bool ok = true;
        for (int t = 0; t < nt; ++t, ++g) {
          const uint32_t st = g % S::STAGES;
          if (!mbar_wait(&b_empty[st], ((g / S::STAGES) & 1) ^ 1, abort_flag, p.status, 11)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&b_full[st], S::B_BYTES);
          for (int ch = 0; ch < S::CH; ++ch)
            tma_load_2d(sB + st * S::B_BYTES + ch * kKeys * S::SWB, &tm_k, &b_full[st],
                        ch * S::CHE, static_cast<int>(mt.key0) + t * kKeys);
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kKeys, 0, 0);
      uint32_t g = 0, acnt = 0, ua = 0;
      for (int round = 0;; ++round) {
        const int u = unit_of(round, cta, nctas);
        if (u >= p.n_mtiles || *abort_flag) break;
        const int nt = mtile_ntiles(p, mtile_of(p, u));
        if (nt == 0) continue;
        if (!mbar_wait(a_full, ua & 1, abort_flag, p.status, 20)) break;
        tc_fence_after();
        bool ok = true;
        for (int t = 0; t < nt; ++t, ++g, ++acnt) {
          const uint32_t st = g % S::STAGES;
          if (!mbar_wait(&b_full[st], (g / S::STAGES) & 1, abort_flag, p.status, 21)) {
            ok = false;
            break;
          }
          const uint32_t acc = acnt & 1;
          if (!mbar_wait(&acc_empty[acc], ((acnt >> 1) & 1) ^ 1, abort_flag, p.status, 22)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * kKeys;
          const uint32_t a_base = smem_u32(sA);
          const uint32_t b_base = smem_u32(sB + st * S::B_BYTES);
#pragma unroll
          for (int ch = 0; ch < S::CH; ++ch) {
#pragma unroll
            for (int s = 0; s < S::KSTEPS; ++s) {
              const uint64_t ad =
                  umma_desc(a_base + ch * kRows * S::SWB + s * 32, 16, S::SBO, S::SWZ);
              const uint64_t bd =
                  umma_desc(b_base + ch * kKeys * S::SWB + s * 32, 16, S::SBO, S::SWZ);
              umma_bf16(d_tmem, ad, bd, idesc, (ch | s) != 0);
            }
          }
          umma_commit(&b_empty[st]);
          umma_commit(&acc_full[acc]);
        }
        if (!ok) break;
        umma_commit(a_empty);
        ++ua;
      }
    }
  } else {
    // ---------------------------------------------------------- epilogue --
    const int grp = (warp - 2) >> 2;          // column half of every key tile
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;      // TMEM lane = row of the M-tile
    const int hcol = grp * kRows + row;       // this thread's column of keys[]
    const int per_half = kHalf / p.B_k;       // blocks per half tile (1 or 2)
    uint32_t acnt = 0, ucnt = 0;
    for (int round = 0;; ++round, ++ucnt) {
      const int u = unit_of(round, cta, nctas);
      if (u >= p.n_mtiles || *abort_flag) break;
      const MTile mt = mtile_of(p, u);
      const int c = mt.c;
      const int nt = mtile_ntiles(p, mt);
      // group 1 reuses its keys[] column once group 0 has merged the last unit
      if (grp == 1 && ucnt > 0 &&
          !mbar_wait(xch_empty, (ucnt - 1) & 1, abort_flag, p.status, 31))
        break;
      // running Top-(k-1): register list (descending; slots before RL-HS hold
      // +inf sentinels that never move) or shared-memory heap
      constexpr int RL = 15;
      float lv[RL];
      int li[RL];
      if constexpr (REG) {
#pragma unroll
        for (int s = 0; s < RL; ++s) {
          lv[s] = s < RL - HS ? INFINITY : -INFINITY;
          li[s] = -1;
        }
      } else {
        for (int s = 0; s < HS; ++s) keys[s * kEpiThreads + hcol] = 0ull;
      }
      float root = HS > 0 ? -INFINITY : INFINITY;
      bool ok = true;
      for (int t = 0; t < nt; ++t, ++acnt) {
        const uint32_t acc = acnt & 1;
        if (!mbar_wait(&acc_full[acc], (acnt >> 1) & 1, abort_flag, p.status, 30)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the row's 128 scores of this half in two steps of 64 columns: the
        // first is reduced before the second is loaded, which keeps the peak
        // register use low enough for the running Top-k list
        const uint32_t ta = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                            acc * kKeys + grp * kHalf;
        float x0, x1, x2, x3;
        {
          uint32_t ra[32], rb[32];
          tmem_ld32(ta + 0, ra);
          tmem_ld32(ta + 32, rb);
          tmem_wait_ld();
          x0 = __uint_as_float(ra[0]);
          x1 = __uint_as_float(rb[0]);
#pragma unroll
          for (int j = 1; j < 31; j += 2) {
            x0 = fmax3(x0, __uint_as_float(ra[j]), __uint_as_float(ra[j + 1]));
            x1 = fmax3(x1, __uint_as_float(rb[j]), __uint_as_float(rb[j + 1]));
          }
          x0 = fmaxf(x0, __uint_as_float(ra[31]));
          x1 = fmaxf(x1, __uint_as_float(rb[31]));
          tmem_ld32(ta + 64, ra);
          tmem_ld32(ta + 96, rb);
          tmem_wait_ld();
          x2 = __uint_as_float(ra[0]);
          x3 = __uint_as_float(rb[0]);
#pragma unroll
          for (int j = 1; j < 31; j += 2) {
            x2 = fmax3(x2, __uint_as_float(ra[j]), __uint_as_float(ra[j + 1]));
            x3 = fmax3(x3, __uint_as_float(rb[j]), __uint_as_float(rb[j + 1]));
          }
          x2 = fmaxf(x2, __uint_as_float(ra[31]));
          x3 = fmaxf(x3, __uint_as_float(rb[31]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        float mx[2];
        if (per_half == 1) {
          mx[0] = fmax3(x0, x1, fmaxf(x2, x3));
          mx[1] = -INFINITY;
        } else {
          mx[0] = fmaxf(x0, x1);
          mx[1] = fmaxf(x2, x3);
        }
        for (int h = 0; h < per_half; ++h) {
          const int b = (2 * t + grp) * per_half + h;
          if constexpr (REG) {
            // a candidate enters only above the last kept score (strict: an
            // equal score belongs to a lower, earlier block, which stays)
            const float x = b < c ? mx[h] : -INFINITY;
            if (!__any_sync(0xFFFFFFFFu, x > lv[RL - 1])) continue;
            bool cmp[RL];
#pragma unroll
            for (int s2 = 0; s2 < RL; ++s2) cmp[s2] = x > lv[s2];
#pragma unroll
            for (int s2 = RL - 1; s2 > 0; --s2) {
              lv[s2] = cmp[s2 - 1] ? lv[s2 - 1] : (cmp[s2] ? x : lv[s2]);
              li[s2] = cmp[s2 - 1] ? li[s2 - 1] : (cmp[s2] ? b : li[s2]);
            }
            lv[0] = cmp[0] ? x : lv[0];
            li[0] = cmp[0] ? b : li[0];
          } else {
            if (b >= c || !(mx[h] > root)) continue;
            // replace the root (worst kept) and sift down; ties -> lower block
            const uint64_t key = pack_key(mx[h], b);
            int pos = 0;
            while (true) {
              const int c1i = 2 * pos + 1;
              if (c1i >= HS) break;
              uint64_t km = keys[c1i * kEpiThreads + hcol];
              int cm = c1i;
              if (c1i + 1 < HS) {
                const uint64_t k2 = keys[(c1i + 1) * kEpiThreads + hcol];
                if (k2 < km) {
                  km = k2;
                  cm = c1i + 1;
                }
              }
              if (km >= key) break;
              keys[pos * kEpiThreads + hcol] = km;
              pos = cm;
            }
            keys[pos * kEpiThreads + hcol] = key;
            root = unorder_key(keys[hcol]);
          }
        }
      }
      if (!ok) break;
      // ---------------------------------- hand over, merge, write the row --
      if constexpr (REG) {
        // the register list as keys, best first
#pragma unroll
        for (int s = 0; s < RL; ++s)
          if (s >= RL - HS)
            keys[(s - (RL - HS)) * kEpiThreads + hcol] = li[s] >= 0 ? pack_key(lv[s], li[s]) : 0ull;
      }
      if (grp == 1) {
        __syncwarp();
        if (lane == 0) mbar_arrive(xch_full);
        continue;
      }
      if (!mbar_wait(xch_full, ucnt & 1, abort_flag, p.status, 32)) break;
      int sel[32];
      float scr[32];  // raw (unscaled) block scores; the local block's is written elsewhere
      int n = 0;
      scr[n] = 0.0f;
      sel[n++] = c;  // the local block (Eq. 7: always kept)
      if constexpr (REG) {
        // both lists are sorted best first: a two-way merge
        int ia = 0, ib = 0;
        for (int s = 0; s < HS; ++s) {
          const uint64_t ka = ia < HS ? keys[ia * kEpiThreads + row] : 0ull;
          const uint64_t kb = ib < HS ? keys[ib * kEpiThreads + kRows + row] : 0ull;
          const uint64_t kbest = ka >= kb ? ka : kb;
          if (kbest == 0ull) break;
          if (ka >= kb) ++ia;
          else ++ib;
          scr[n] = unorder_key(kbest);
          sel[n++] = key_block(kbest);
        }
      } else {
        // two heaps: take the best remaining key HS times
        uint64_t taken_below = ~0ull;  // keys are distinct, so "below the last taken"
        for (int s = 0; s < HS; ++s) {
          uint64_t best = 0ull;
          for (int j = 0; j < 2 * HS; ++j) {
            const uint64_t kj = keys[(j % HS) * kEpiThreads + (j / HS) * kRows + row];
            if (kj < taken_below && kj > best) best = kj;
          }
          if (best == 0ull) break;
          taken_below = best;
          scr[n] = unorder_key(best);
          sel[n++] = key_block(best);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xch_empty);
      const int64_t row_glob = mt.row0 + row;
      if (row < mt.nrows) {
        for (int a = 1; a < n; ++a) {  // ascending
          const int x = sel[a];
          const float xs = scr[a];
          int b = a - 1;
          while (b >= 0 && sel[b] > x) {
            sel[b + 1] = sel[b];
            scr[b + 1] = scr[b];
            --b;
          }
          sel[b + 1] = x;
          scr[b + 1] = xs;
        }
        int32_t* out = p.idx_out + row_glob * p.k;
        for (int s = 0; s < p.k; ++s) out[s] = s < n ? sel[s] : -1;
        if (p.score_out != nullptr) {
          // the local block (the largest index, so slot n - 1) is scored by
          // local_block_score_kernel
          float* so = p.score_out + row_glob * p.k;
          for (int s = 0; s < p.k; ++s)
            if (s != n - 1) so[s] = s < n ? scr[s] * p.scale : -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// score_out of each row's local block (its last valid slot, min(k, b_i + 1)
// - 1): the Eq. 6 maximum over the block's keys j <= i, one warp per (query,
// group), lane l scoring keys l, l + 32, ... of the block.
template <int D_IDX>
__global__ void __launch_bounds__(256) local_block_score_kernel(const __nv_bfloat16* q_idx,
                                                                const __nv_bfloat16* k_idx,
                                                                const IndexParams p) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= p.N * p.H_kv) return;
  const int64_t i = row / p.H_kv;
  const int64_t i0 = p.qinfo != nullptr ? p.qinfo[i].x : 0;  // first token of i's sequence
  const int64_t b_i = (i - i0) / p.B_k;
  float q[D_IDX];
  const __nv_bfloat16* qr = q_idx + row * D_IDX;
#pragma unroll
  for (int d = 0; d < D_IDX; d += 2) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qr + d));
    q[d] = f.x;
    q[d + 1] = f.y;
  }
  float m = -INFINITY;
  for (int64_t j = i0 + b_i * p.B_k + lane; j <= i; j += 32) {
    const __nv_bfloat16* kr = k_idx + j * D_IDX;
    float dot = 0.0f;
#pragma unroll
    for (int d = 0; d < D_IDX; d += 8) {
      const uint4 w = *reinterpret_cast<const uint4*>(kr + d);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h[e]);
        dot = fmaf(q[d + 2 * e], f.x, dot);
        dot = fmaf(q[d + 2 * e + 1], f.y, dot);
      }
    }
    m = fmaxf(m, dot);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if (lane == 0) {
    const int64_t slot = (b_i + 1 < p.k ? b_i + 1 : p.k) - 1;
    p.score_out[row * p.k + slot] = m * p.scale;
  }
}

template <int D_IDX>
size_t index_smem_bytes(int k) {
  using S = IndexShape<D_IDX>;
  const int hs = k - 1 > 0 ? k - 1 : 1;
  return 1024 + S::A_BYTES + S::STAGES * S::B_BYTES + static_cast<size_t>(kEpiThreads) * hs * 8 +
         (2 + 2 * S::STAGES + 4 + 2) * 8 + 16;
}

template <int D_IDX>
cudaError_t launch_typed(const IndexLaunch& a, cudaStream_t stream) {
  using S = IndexShape<D_IDX>;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D_IDX), static_cast<uint64_t>(a.N) * a.H_kv};
    const uint64_t strides[1] = {static_cast<uint64_t>(D_IDX) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(S::CHE), static_cast<uint32_t>(kRows)};
    if (!make_tmap_bf16(&tq, a.q_idx, 2, dims, strides, box, S::SWB)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(D_IDX), static_cast<uint64_t>(a.N)};
    const uint64_t strides[1] = {static_cast<uint64_t>(D_IDX) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(S::CHE), static_cast<uint32_t>(kKeys)};
    if (!make_tmap_bf16(&tk, a.k_idx, 2, dims, strides, box, S::SWB)) return cudaErrorInvalidValue;
  }
  IndexParams p;
  p.N = a.N;
  p.H_kv = a.H_kv;
  p.B_k = a.B_k;
  p.k = a.k;
  p.n_mtiles = a.tiles != nullptr ? a.n_tiles
                                  : static_cast<int>((a.N * a.H_kv + kRows - 1) / kRows);
  p.tiles = a.tiles;
  p.qinfo = a.qinfo;
  p.idx_out = a.idx_out;
  p.score_out = a.score_out;
  p.scale = a.scale;
  p.status = a.status;
  const bool reg = a.k <= 16;
  const size_t smem = index_smem_bytes<D_IDX>(a.k);
  auto kern = reg ? index_topk_kernel<D_IDX, true> : index_topk_kernel<D_IDX, false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int grid = num_sms();
  if (grid > p.n_mtiles) grid = p.n_mtiles;
  if (grid < 1) grid = 1;
  prof_begin("index_topk", stream);
  kern<<<grid, kThreads, smem, stream>>>(tq, tk, p);
  prof_end(stream);
  if (a.score_out != nullptr) {
    const int64_t threads = a.N * a.H_kv * 32;
    prof_begin("local_block_score", stream);
    local_block_score_kernel<D_IDX><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(a.q_idx), static_cast<const __nv_bfloat16*>(a.k_idx), p);
    prof_end(stream);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_topk(const IndexLaunch& a, cudaStream_t s) {
  switch (a.d_idx) {
    case 32: return launch_typed<32>(a, s);
    case 64: return launch_typed<64>(a, s);
    case 128: return launch_typed<128>(a, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace msa
