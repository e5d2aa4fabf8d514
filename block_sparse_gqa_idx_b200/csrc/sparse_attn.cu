// sparse_attn.cu -- Main Branch (Eq. 8 with the causal rule of Eq. 1) as a
// KV-outer block-sparse attention on tcgen05, in three steps per query chunk:
//
//   1. inverse index (inv_index.cu): for every (group r, block b) the list
//      of selection slots that chose b, cut into tiles of Tq queries
//      (Tq * rows-per-query = 128 MMA rows) with every output slot fixed.
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
// Source: xllm-io paper review, "核心公式" Eq. 8 and "4.2 Sparse Attention
// Kernel" (KV-outer with query gather, two-phase forward: partial outputs
// then a combine pass); chlience notes 5.4 (pre-scheduled tile chunking,
// slots assigned ahead, two-phase combine).
#include <climits>
#include <type_traits>

#include "attn_common.cuh"

namespace msa {
namespace {

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
      // scale, exponent, row sums and 1/l on packed pairs of a row's two keys
      // (the halves of lA2 and lB2 are the row's two running sums)
      const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
      const uint64_t nmA = f2_pack(-msA, -msA), nmB = f2_pack(-msB, -msB);
      uint64_t lA2 = f2_pack(0.0f, 0.0f), lB2 = lA2;
#pragma unroll
      for (int r = 0; r < B_K / 8; ++r) {
        const uint64_t xa = f2_fma(
            f2_pack(__uint_as_float(v[4 * r]), __uint_as_float(v[4 * r + 1])), sc2, nmA);
        const uint64_t xb = f2_fma(
            f2_pack(__uint_as_float(v[4 * r + 2]), __uint_as_float(v[4 * r + 3])), sc2, nmB);
        const float a0 = ex2_ftz(f2_lo(xa)), a1 = ex2_ftz(f2_hi(xa));
        const float b0 = ex2_ftz(f2_lo(xb)), b1 = ex2_ftz(f2_hi(xb));
        lA2 = f2_add(lA2, f2_pack(a0, a1));
        lB2 = f2_add(lB2, f2_pack(b0, b1));
        v[4 * r] = __float_as_uint(a0);
        v[4 * r + 1] = __float_as_uint(a1);
        v[4 * r + 2] = __float_as_uint(b0);
        v[4 * r + 3] = __float_as_uint(b1);
      }
      float lA = f2_lo(lA2) + f2_hi(lA2), lB = f2_lo(lB2) + f2_hi(lB2);
#pragma unroll
      for (int o = 1; o < 4; o <<= 1) {
        lA += __shfl_xor_sync(0xFFFFFFFFu, lA, o);
        lB += __shfl_xor_sync(0xFFFFFFFFu, lB, o);
      }
      const float invA = 1.0f / lA, invB = 1.0f / lB;
      const uint64_t invA2 = f2_pack(invA, invA), invB2 = f2_pack(invB, invB);
      // P / l as bf16 pairs: the pair of keys (8r + 2c, 8r + 2c + 1) is P
      // column 4r + c
      uint32_t pk[B_K / 4];
#pragma unroll
      for (int r = 0; r < B_K / 8; ++r) {
        const uint64_t na = f2_mul(
            f2_pack(__uint_as_float(v[4 * r]), __uint_as_float(v[4 * r + 1])), invA2);
        const uint64_t nb = f2_mul(
            f2_pack(__uint_as_float(v[4 * r + 2]), __uint_as_float(v[4 * r + 3])), invB2);
        __nv_bfloat162 xa = __floats2bfloat162_rn(f2_lo(na), f2_hi(na));
        __nv_bfloat162 xb = __floats2bfloat162_rn(f2_lo(nb), f2_hi(nb));
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
  // this lane's head: the largest LSE of its used slots.  All of the row's
  // LSEs are loaded together with the selection (a slot that turns out
  // unused is never read into the arithmetic), then kept in registers only
  // for the maximum; the weights read them again below, from L1.
  const float* lse_h = p.c.part_lse + slot0 * p.G + g;
  float lv[32];
#pragma unroll
  for (int s = 0; s < 32; ++s) lv[s] = s < p.kk ? lse_h[s * p.G] : -INFINITY;
  const unsigned use = __ballot_sync(0xFFFFFFFFu, lane < p.kk && myb >= 0 && myb <= b_i);
  float m = -INFINITY;
#pragma unroll
  for (int s = 0; s < 32; ++s) m = ((use >> s) & 1u) ? fmaxf(m, lv[s]) : m;
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

}  // namespace

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

}  // namespace msa
