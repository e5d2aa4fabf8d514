// decode.cu -- one MSA decode step for S independent sequences.
//
// Per sequence s with L = seq_len[s]:
//   scan     append k/v/k_idx of the new token at row L (Eq. 1: the query
//            sees i <= t, itself included), then Eq. 6 for the single query
//            i = L over the full blocks 0..b_i-1
//            (b_i = L / B_k; the local block b_i is forced and needs no score):
//            block maxima of the H_kv index-query dots, streamed from the K_idx
//            cache.  HBM-bound: 2*d_idx bytes per cached token.
//   top-k    Eq. 7: one warp per (s, r) keeps per-lane sorted candidate lists
//            and merges them in k-1 warp-argmax rounds (ties -> lower block).
//   attend   Eq. 8: one CTA per (s, r, slot) gathers that block's K/V rows
//            (TMA), S = q K^T and O = P V on mma.sync, causal mask j <= L in
//            the local block; writes a normalised partial and its LSE.
//   merge    LSE-weighted combine of the <= k partials per head; seq_len += 1.
//
// Source: xllm-io paper review, "核心公式" Eq. 1, 6, 7, 8; chlience notes
// 5.1.1 (selection steps) and 5.4 (exp-free selection on raw scores).
#include <atomic>

#include <cuda.h>
#include <cuda_runtime.h>

#include <cuda_fp8.h>

#include "msa_internal.h"

namespace msa {
namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct DecBufs {
  int32_t* Lcur;    // [S] this step's length before the append, -1 = skipped
  float* M;         // [S, H_kv, Bmax] block maxima (raw dots)
  int32_t* sel;     // [S, H_kv, k]
  float* part_o;    // [S, H_kv, k, G, d_h] normalised partial outputs
  float* part_lse;  // [S, H_kv, k, G]
};

DecBufs carve(void* ws, int S, int64_t L_max, int H_q, int H_kv, int d_h, int B_k, int kk,
              size_t* total) {
  DecBufs b;
  uint8_t* p = static_cast<uint8_t*>(ws);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* r = p ? p + off : nullptr;
    off += align256(bytes);
    return r;
  };
  const int64_t Bmax = (L_max + B_k - 1) / B_k + 1;
  const int G = H_q / H_kv;
  b.Lcur = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * S));
  b.M = reinterpret_cast<float*>(take(sizeof(float) * S * H_kv * Bmax));
  b.sel = reinterpret_cast<int32_t*>(take(sizeof(int32_t) * S * H_kv * kk));
  b.part_o = reinterpret_cast<float*>(take(sizeof(float) * S * H_kv * kk * G * d_h));
  b.part_lse = reinterpret_cast<float*>(take(sizeof(float) * S * H_kv * kk * G));
  *total = off;
  return b;
}

struct DecParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* q_idx;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const __nv_bfloat16* k_idx_new;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  __nv_bfloat16* k_idx_cache;
  int32_t* seq_len;
  __nv_bfloat16* o;
  int32_t* idx_out;
  int S;
  int64_t L_max, Bmax;
  int H_q, H_kv, d_h, d_idx, B_k, kk, G;
  float scale_log2, scale;
  DecBufs w;
  DevStatus* status;
};

// -------------------------------------------------------------------- scan --
// One warp scores one 128-key block at a time (B_k = 128: 8 row tiles of 16
// keys; B_k = 64: 4).  MMA rows = keys, columns = index-query heads (padded
// to 8), reduction over d_idx.  The d axis is consumed in a per-thread order
// (thread t of a quad owns d in [t*D/4, (t+1)*D/4)), applied identically to
// the A rows (keys, loaded straight from global memory with 16-byte loads)
// and to the B columns (index queries), so every dot product is complete.
template <int D_IDX, int BK>
__global__ void __launch_bounds__(256) dec_scan_kernel(const DecParams p, int nsplit) {
  constexpr int DT = D_IDX / 4;       // d elements per thread and key row
  constexpr int NMMA = D_IDX / 16;    // MMAs per 16-key tile
  constexpr int NV = DT / 8;          // 16-byte loads per key row
  const int s = blockIdx.y;
  const int64_t L = p.seq_len[s];  // written back (L + 1) only by the merge kernel
  if (L < 0 || L >= p.L_max) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.w.Lcur[s] = -1;
      report(p.status, DEV_ERR_CACHE_FULL, 80, s, static_cast<int>(L));
    }
    return;
  }
  if (blockIdx.x == 0) {
    // append the new token's rows at position L (the scan below never reads
    // them: they lie in the local block, which is forced, not scored)
    const int kv16 = p.H_kv * p.d_h / 8;  // 16-byte pieces per K (or V) row
    const uint4* kn = reinterpret_cast<const uint4*>(p.k_new + static_cast<int64_t>(s) * p.H_kv * p.d_h);
    const uint4* vn = reinterpret_cast<const uint4*>(p.v_new + static_cast<int64_t>(s) * p.H_kv * p.d_h);
    const uint4* kin = reinterpret_cast<const uint4*>(p.k_idx_new + static_cast<int64_t>(s) * D_IDX);
    uint4* kc = reinterpret_cast<uint4*>(p.k_cache + (s * p.L_max + L) * p.H_kv * p.d_h);
    uint4* vc = reinterpret_cast<uint4*>(p.v_cache + (s * p.L_max + L) * p.H_kv * p.d_h);
    uint4* kic = reinterpret_cast<uint4*>(p.k_idx_cache + (s * p.L_max + L) * D_IDX);
    for (int t = threadIdx.x; t < kv16; t += blockDim.x) {
      kc[t] = kn[t];
      vc[t] = vn[t];
    }
    for (int t = threadIdx.x; t < D_IDX / 8; t += blockDim.x) kic[t] = kin[t];
    if (threadIdx.x == 0) p.w.Lcur[s] = static_cast<int32_t>(L);
  }
  const int64_t b_i = L / p.B_k;  // candidate blocks 0 .. b_i-1
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  // B fragments: column n = g (index-query head), k-slots follow the d order.
  uint32_t bq[NMMA][2];
  {
    const __nv_bfloat16* qr = p.q_idx + (static_cast<int64_t>(s) * p.H_kv + (g < p.H_kv ? g : 0)) * D_IDX;
#pragma unroll
    for (int j = 0; j < NMMA; ++j) {
      const int d0 = t * DT + 4 * j;
      uint32_t lo = *reinterpret_cast<const uint32_t*>(qr + d0);
      uint32_t hi = *reinterpret_cast<const uint32_t*>(qr + d0 + 2);
      bq[j][0] = g < p.H_kv ? lo : 0u;
      bq[j][1] = g < p.H_kv ? hi : 0u;
    }
  }
  const __nv_bfloat16* kbase = p.k_idx_cache + static_cast<int64_t>(s) * p.L_max * D_IDX;
  const int wstride = nsplit * 8;
  for (int64_t b = blockIdx.x * 8 + warp; b < b_i; b += wstride) {
    float mx0 = -INFINITY, mx1 = -INFINITY;  // columns 2t, 2t+1
#pragma unroll
    for (int tile = 0; tile < BK / 16; ++tile) {
      const __nv_bfloat16* r0 = kbase + (b * BK + tile * 16 + g) * D_IDX + t * DT;
      const __nv_bfloat16* r1 = r0 + 8 * D_IDX;
      uint4 v0[NV], v1[NV];
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        v0[u] = __ldg(reinterpret_cast<const uint4*>(r0) + u);
        v1[u] = __ldg(reinterpret_cast<const uint4*>(r1) + u);
      }
      const uint32_t* w0 = reinterpret_cast<const uint32_t*>(v0);
      const uint32_t* w1 = reinterpret_cast<const uint32_t*>(v1);
      float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < NMMA; ++j) {
        // k-slots 2t,2t+1 <- d0,d0+1 ; 2t+8,2t+9 <- d0+2,d0+3 (d0 = t*DT + 4j)
        const uint32_t a[4] = {w0[2 * j], w1[2 * j], w0[2 * j + 1], w1[2 * j + 1]};
        mma_bf16_16816(c, a, bq[j][0], bq[j][1]);
      }
      mx0 = fmax3(mx0, c[0], c[2]);
      mx1 = fmax3(mx1, c[1], c[3]);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o));
    }
    if (g == 0) {
      const int r0 = 2 * t, r1 = 2 * t + 1;
      float* Mrow = p.w.M + static_cast<int64_t>(s) * p.H_kv * p.Bmax;
      if (r0 < p.H_kv) Mrow[r0 * p.Bmax + b] = mx0;
      if (r1 < p.H_kv) Mrow[r1 * p.Bmax + b] = mx1;
    }
  }
}

// ------------------------------------------------------------------- top-k --
__device__ __forceinline__ uint64_t pack_key(float v, int b) {
  uint32_t u = __float_as_uint(v);
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(b));
}

// One CTA (8 warps) per (sequence, group).  Warp w scans blocks w*32+lane,
// +256, ... keeping per-lane sorted lists in shared memory, and reduces them
// to its best k-1 in k-1 rounds of warp argmax.  Warp 0 then ranks the 8
// warps' winners against each other (count of larger keys), keeps the k-1
// best, adds the local block and writes the set in ascending block order.
__global__ void __launch_bounds__(256) dec_topk_kernel(const DecParams p) {
  griddep_wait();  // the previous kernel of the step has finished
  extern __shared__ uint64_t lists[];  // [8 warps][k-1][32 lanes] + winners [8][k-1]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int s = pair / p.H_kv, r = pair - s * p.H_kv;
  const int64_t L = p.w.Lcur[s];
  if (L < 0) return;
  const int b_i = static_cast<int>(L / p.B_k);
  const int HS = p.kk - 1;
  const int hs1 = HS > 0 ? HS : 1;
  uint64_t* my = lists + static_cast<size_t>(warp) * hs1 * 32;
  uint64_t* win = lists + static_cast<size_t>(8) * hs1 * 32;  // [8][hs1]
  __shared__ int32_t chosen[33];
  const float* Mrow = p.w.M + (static_cast<int64_t>(s) * p.H_kv + r) * p.Bmax;
  int cnt = 0;
  uint64_t worst = 0;  // smallest kept key once the list is full
  for (int b = warp * 32 + lane; b < b_i && HS > 0; b += 256) {
    const uint64_t key = pack_key(Mrow[b], b);
    if (cnt == HS && key <= worst) continue;
    int pos = cnt < HS ? cnt : HS - 1;
    while (pos > 0 && my[(pos - 1) * 32 + lane] < key) {
      my[pos * 32 + lane] = my[(pos - 1) * 32 + lane];
      --pos;
    }
    my[pos * 32 + lane] = key;
    if (cnt < HS) ++cnt;
    worst = my[(cnt - 1) * 32 + lane];
  }
  // this warp's best HS keys (0 = none), by rounds of warp argmax
  int head = 0;
  for (int round = 0; round < HS; ++round) {
    const uint64_t cand = head < cnt ? my[head * 32 + lane] : 0ull;
    uint64_t best = cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, best, o);
      best = other > best ? other : best;
    }
    if (cand == best && cand != 0ull) ++head;
    if (lane == 0) win[warp * hs1 + round] = best;
  }
  __syncthreads();
  // rank the 8 warps' winners, one thread per winner: a key is kept if fewer
  // than HS keys beat it (keys are distinct: each carries its block)
  const int T = 8 * HS;
  bool keep = false;
  if (static_cast<int>(threadIdx.x) < T) {
    const uint64_t mine = win[threadIdx.x];
    int rank = 0;
    if (mine != 0ull)
      for (int m = 0; m < T; ++m) rank += win[m] > mine ? 1 : 0;
    keep = mine != 0ull && rank < HS;
    if (keep) chosen[rank] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(mine));
  }
  const int nkept = __syncthreads_count(keep);
  if (warp != 0) return;
  if (lane == 0) chosen[nkept] = b_i;  // the local block (Eq. 7: always kept)
  __syncwarp();
  const int nsel = nkept + 1;
  const int32_t v = lane < nsel ? chosen[lane] : -1;
  int pos = 0;
  for (int m = 0; m < nsel; ++m) pos += chosen[m] < v ? 1 : 0;
  int32_t* dst = p.w.sel + (static_cast<int64_t>(s) * p.H_kv + r) * p.kk;
  int32_t* dst2 = p.idx_out != nullptr ? p.idx_out + (static_cast<int64_t>(s) * p.H_kv + r) * p.kk : nullptr;
  if (lane < nsel) {
    dst[pos] = v;
    if (dst2) dst2[pos] = v;
  } else if (lane < p.kk) {
    dst[lane] = -1;
    if (dst2) dst2[lane] = -1;
  }
}

// ------------------------------------------------------------------ attend --
// Byte address of (row, 16-byte chunk c) in a TMA tile of 128-byte rows with
// 128-byte swizzle (chunks XOR row mod 8), split in 64-element column boxes.
template <int BK>
__device__ __forceinline__ uint32_t sw_addr(uint32_t base, int row, int d) {
  const int box = d >> 6, c = (d >> 3) & 7;
  return base + box * BK * 128 + row * 128 + ((c ^ (row & 7)) << 4);
}

// One CTA (4 warps) per (sequence, group, slot).  Rows of the MMA are the
// group's query heads (G <= 16, padded to 16); warp w owns keys
// [w*BK/4, (w+1)*BK/4) of the block; the four partial softmax states are
// merged through shared memory.
template <int D_H, int BK>
__global__ void __launch_bounds__(128) dec_attend_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                         const __grid_constant__ CUtensorMap tm_v,
                                                         const DecParams p) {
  griddep_wait();  // the previous kernel of the step has finished
  constexpr int KW = BK / 4;          // keys per warp
  constexpr int NT = KW / 8;          // S n-tiles per warp
  constexpr int DT = D_H / 8;         // O n-tiles
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + BK * D_H * 2;
  float* red = reinterpret_cast<float*>(sV + BK * D_H * 2);  // [4][16] m, [4][16] l
  uint64_t* bar = reinterpret_cast<uint64_t*>(red + 128);    // [0] K landed, [1] V landed
  float* obuf = reinterpret_cast<float*>(smem);  // [4][16][D_H], over K/V once both are used

  const int item = blockIdx.x;  // (s, r, slot)
  const int slot = item % p.kk;
  const int r = (item / p.kk) % p.H_kv;
  const int s = item / (p.kk * p.H_kv);
  const int64_t L = p.w.Lcur[s];
  if (L < 0) return;
  const int b = p.w.sel[(static_cast<int64_t>(s) * p.H_kv + r) * p.kk + slot];
  if (b < 0) return;
  const int64_t last = L;  // the new token's position: keys j <= last
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int row0 = static_cast<int>(s * p.L_max + static_cast<int64_t>(b) * BK);
    mbar_arrive_expect_tx(&bar[0], BK * D_H * 2);
    for (int c = 0; c < D_H / 64; ++c) tma_load_3d(sK + c * BK * 128, &tm_k, &bar[0], c * 64, r, row0);
    mbar_arrive_expect_tx(&bar[1], BK * D_H * 2);
    for (int c = 0; c < D_H / 64; ++c) tma_load_3d(sV + c * BK * 128, &tm_v, &bar[1], c * 64, r, row0);
  }
  // Q fragments (rows = heads, zero beyond G) while the tiles land.
  uint32_t qa[D_H / 16][4];
  {
    const __nv_bfloat16* qb = p.q + (static_cast<int64_t>(s) * p.H_q + r * p.G) * D_H;
#pragma unroll
    for (int ks = 0; ks < D_H / 16; ++ks) {
      const int d = ks * 16 + 2 * t;
      qa[ks][0] = g < p.G ? *reinterpret_cast<const uint32_t*>(qb + g * D_H + d) : 0u;
      qa[ks][1] = g + 8 < p.G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D_H + d) : 0u;
      qa[ks][2] = g < p.G ? *reinterpret_cast<const uint32_t*>(qb + g * D_H + d + 8) : 0u;
      qa[ks][3] = g + 8 < p.G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D_H + d + 8) : 0u;
    }
  }
  bool ok = mbar_wait(&bar[0], 0, nullptr, p.status, 90);
  const int kw0 = warp * KW;  // first key (within the block) of this warp
  float sacc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
  if (ok) {
    const uint32_t kb = smem_u32(sK);
#pragma unroll
    for (int ks = 0; ks < D_H / 16; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2) {
        // matrices: (keys 0-7, d lo), (keys 0-7, d hi), (keys 8-15, d lo), (keys 8-15, d hi)
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kw0 + n2 * 16 + (mi >> 1) * 8 + rr;
        const int d = ks * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sw_addr<BK>(kb, key, d), b0, b1, b2, b3);
        mma_bf16_16816(sacc[2 * n2], qa[ks], b0, b1);
        mma_bf16_16816(sacc[2 * n2 + 1], qa[ks], b2, b3);
      }
    }
  }
  // scale, causal mask (only the block holding the new token), row max / sum
  const int64_t j0 = static_cast<int64_t>(b) * BK + kw0;
  float m_lo = -INFINITY, m_hi = -INFINITY;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t j = j0 + n * 8 + 2 * t + (e & 1);
      float x = sacc[n][e] * p.scale_log2;
      if (j > last) x = -INFINITY;
      sacc[n][e] = x;
    }
    m_lo = fmax3(m_lo, sacc[n][0], sacc[n][1]);
    m_hi = fmax3(m_hi, sacc[n][2], sacc[n][3]);
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    m_lo = fmaxf(m_lo, __shfl_xor_sync(0xFFFFFFFFu, m_lo, o));
    m_hi = fmaxf(m_hi, __shfl_xor_sync(0xFFFFFFFFu, m_hi, o));
  }
  const float ms_lo = m_lo == -INFINITY ? 0.f : m_lo;
  const float ms_hi = m_hi == -INFINITY ? 0.f : m_hi;
  float l_lo = 0.f, l_hi = 0.f;
  uint32_t pa[NT / 2][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float e0 = exp2f(sacc[n][0] - ms_lo), e1 = exp2f(sacc[n][1] - ms_lo);
    const float e2 = exp2f(sacc[n][2] - ms_hi), e3 = exp2f(sacc[n][3] - ms_hi);
    l_lo += e0 + e1;
    l_hi += e2 + e3;
    // A fragment of P for k-step n/2: n even -> regs 0,1 ; n odd -> regs 2,3
    pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(e0, e1);
    pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(e2, e3);
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    l_lo += __shfl_xor_sync(0xFFFFFFFFu, l_lo, o);
    l_hi += __shfl_xor_sync(0xFFFFFFFFu, l_hi, o);
  }
  float oacc[DT][4];
#pragma unroll
  for (int n = 0; n < DT; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  ok = ok && mbar_wait(&bar[1], 0, nullptr, p.status, 91);
  if (ok) {
    const uint32_t vb = smem_u32(sV);
#pragma unroll
    for (int ks = 0; ks < NT / 2; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < DT / 2; ++n2) {
        // matrices: (keys 0-7, d lo), (keys 8-15, d lo), (keys 0-7, d hi), (keys 8-15, d hi)
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kw0 + ks * 16 + (mi & 1) * 8 + rr;
        const int d = n2 * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sw_addr<BK>(vb, key, d), b0, b1, b2, b3);
        mma_bf16_16816(oacc[2 * n2], pa[ks], b0, b1);
        mma_bf16_16816(oacc[2 * n2 + 1], pa[ks], b2, b3);
      }
    }
  }
  // merge the four warps' (m, l, O) through shared memory (log2 domain);
  // obuf overlays the K/V tiles, so every warp must be done with them first
  __syncthreads();
  if (t == 0) {
    red[warp * 16 + g] = m_lo;
    red[warp * 16 + g + 8] = m_hi;
    red[64 + warp * 16 + g] = l_lo;
    red[64 + warp * 16 + g + 8] = l_hi;
  }
#pragma unroll
  for (int n = 0; n < DT; ++n) {
    float* o0 = obuf + (warp * 16 + g) * D_H + n * 8 + 2 * t;
    float* o1 = obuf + (warp * 16 + g + 8) * D_H + n * 8 + 2 * t;
    o0[0] = oacc[n][0];
    o0[1] = oacc[n][1];
    o1[0] = oacc[n][2];
    o1[1] = oacc[n][3];
  }
  __syncthreads();
  // thread -> (head row, d slice): 16 rows x 8 threads
  const int hr = threadIdx.x >> 3, part = threadIdx.x & 7;
  if (hr < p.G) {
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red[w * 16 + hr]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float wsum = 0.f, wt[4];
    for (int w = 0; w < 4; ++w) {
      const float mw = red[w * 16 + hr];
      wt[w] = mw == -INFINITY ? 0.f : exp2f(mw - Ms);
      wsum += wt[w] * red[64 + w * 16 + hr];
    }
    const int64_t pslot = ((static_cast<int64_t>(s) * p.H_kv + r) * p.kk + slot) * p.G + hr;
    float* dst = p.w.part_o + pslot * D_H;
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    for (int d = part; d < D_H; d += 8) {
      float acc = 0.f;
      for (int w = 0; w < 4; ++w) acc += wt[w] * obuf[(w * 16 + hr) * D_H + d];
      dst[d] = acc * inv;
    }
    if (part == 0)
      p.w.part_lse[pslot] = wsum > 0.f ? (M + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
  }
}

// ------------------------------------------------------------------- merge --
// One warp per (sequence, head): lane s reads slot s's selection and LSE, the
// weights come from warp reductions, then every slot's partial row (lane:
// D_H/32 consecutive floats) is fetched with all loads in flight.
template <int D_H>
__global__ void __launch_bounds__(256) dec_merge_kernel(const DecParams p) {
  griddep_wait();  // the previous kernel of the step has finished
  constexpr int PER = D_H / 32;
  const int lane = threadIdx.x & 31;
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (s, h)
  if (row >= p.S * p.H_q) return;
  const int s = row / p.H_q, h = row - s * p.H_q;
  const int r = h / p.G, g = h - r * p.G;
  const int64_t L = p.w.Lcur[s];
  if (L < 0) return;
  const int64_t base_slot = (static_cast<int64_t>(s) * p.H_kv + r) * p.kk;
  const bool valid = lane < p.kk && p.w.sel[base_slot + (lane < p.kk ? lane : 0)] >= 0;
  float ls = valid ? p.w.part_lse[(base_slot + lane) * p.G + g] : -INFINITY;
  float m = ls;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  const float w = (valid && ls != -INFINITY) ? __expf(ls - m) : 0.f;
  float wsum = w;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xFFFFFFFFu, wsum, o);
  const unsigned use = __ballot_sync(0xFFFFFFFFu, w > 0.f);
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  const float* src = p.w.part_o + (base_slot * p.G + g) * D_H + lane * PER;
  const int64_t stride = static_cast<int64_t>(p.G) * D_H;
#pragma unroll
  for (int s0 = 0; s0 < 32; s0 += 8) {
    if (s0 >= p.kk) break;
    float x[8][PER];
    float wj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int sl = s0 + j;
      wj[j] = __shfl_sync(0xFFFFFFFFu, w, sl);
      const bool on = (use >> sl) & 1u;
#pragma unroll
      for (int e = 0; e < PER; e += 4) {
        const float4 f = on ? *reinterpret_cast<const float4*>(src + sl * stride + e)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        x[j][e] = f.x;
        x[j][e + 1] = f.y;
        x[j][e + 2] = f.z;
        x[j][e + 3] = f.w;
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(wj[j], x[j][e], acc[e]);
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = p.o + (static_cast<int64_t>(s) * p.H_q + h) * D_H + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2)
    *reinterpret_cast<__nv_bfloat162*>(dst + e) = __floats2bfloat162_rn(acc[e] * inv, acc[e + 1] * inv);
  // seq_len is read only by the scan kernel; the rest of the step uses Lcur
  if (h == 0 && lane == 0) p.seq_len[s] = static_cast<int32_t>(L + 1);
}

template <int D_H, int BK>
size_t attend_smem() {
  static_assert(4 * 16 * D_H * 4 <= 2 * BK * D_H * 2, "warp-merge buffer must fit over K/V");
  return 1024 + 2 * BK * D_H * 2 + 128 * 4 + 16;
}

template <int D_H, int BK>
cudaError_t launch_attend(const DecParams& p, cudaStream_t stream) {
  CUtensorMap tk, tv;
  const uint64_t dims[3] = {static_cast<uint64_t>(D_H), static_cast<uint64_t>(p.H_kv),
                            static_cast<uint64_t>(p.S) * static_cast<uint64_t>(p.L_max)};
  const uint64_t strides[2] = {static_cast<uint64_t>(D_H) * 2,
                               static_cast<uint64_t>(p.H_kv) * D_H * 2};
  const uint32_t box[3] = {64, 1, static_cast<uint32_t>(BK)};
  if (!make_tmap_bf16(&tk, p.k_cache, 3, dims, strides, box, 128)) return cudaErrorInvalidValue;
  if (!make_tmap_bf16(&tv, p.v_cache, 3, dims, strides, box, 128)) return cudaErrorInvalidValue;
  const size_t smem = attend_smem<D_H, BK>();
  cudaError_t e = cudaFuncSetAttribute(dec_attend_kernel<D_H, BK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  prof_begin("dec_attend", stream);
  e = launch_pdl(dec_attend_kernel<D_H, BK>, dim3(p.S * p.H_kv * p.kk), dim3(128), smem, stream,
                 tk, tv, p);
  prof_end(stream);
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int D_IDX>
cudaError_t launch_scan(const DecParams& p, cudaStream_t stream) {
  const int nsplit = p.S >= 64 ? 8 : (p.S >= 16 ? 32 : 64);
  dim3 grid(nsplit, p.S);
  prof_begin("dec_scan", stream);
  if (p.B_k == 128) dec_scan_kernel<D_IDX, 128><<<grid, 256, 0, stream>>>(p, nsplit);
  else dec_scan_kernel<D_IDX, 64><<<grid, 256, 0, stream>>>(p, nsplit);
  prof_end(stream);
  return cudaGetLastError();
}

// ------------------------------------------------- FP8 paged KV-cache decode --
// The same step on a paged cache of E4M3 codes with one float32 scale per
// token (and KV head): value = e4m3(code) * scale.  Logical block b of
// sequence s lives in page page_table[s, b] (pages hold B_k tokens):
//   k_pages, v_pages [P, B_k, H_kv, d_h] codes, k_scale, v_scale [P, B_k, H_kv]
//   kidx_pages [P, B_k, d_idx] codes, kidx_scale [P, B_k]
// Every E4M3 value is exact in bf16, so the kernels feed the codes to the
// bf16 tensor-core paths unchanged and apply the scales in float32: a key's
// scale multiplies its scores, a value's scale multiplies its softmax
// weight before P V.  The append quantizes the new token (amax / 448 per row,
// the division and the E4M3 rounding in float32, saturated).
struct Dec8Params {
  const __nv_bfloat16* q;
  const __nv_bfloat16* q_idx;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const __nv_bfloat16* k_idx_new;
  uint8_t* k_pages;
  float* k_scale;
  uint8_t* v_pages;
  float* v_scale;
  uint8_t* kidx_pages;
  float* kidx_scale;
  const int32_t* page_table;  // [S, max_pages]
  int max_pages;
  int64_t n_pages;
};

// Quantize one row of n bf16 values to E4M3 codes with scale amax / 448 (1
// for an all-zero row), by one warp; returns the scale.
__device__ __forceinline__ float quantize_row_warp(const __nv_bfloat16* x, int n, uint8_t* codes) {
  const int lane = threadIdx.x & 31;
  float amax = 0.0f;
  for (int d = lane; d < n; d += 32) amax = fmaxf(amax, fabsf(__bfloat162float(x[d])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  for (int d = 2 * lane; d < n; d += 64) {
    const float2 y = make_float2(__fdiv_rn(__bfloat162float(x[d]), sc),
                                 __fdiv_rn(__bfloat162float(x[d + 1]), sc));
    const __nv_fp8x2_storage_t c2 = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<uint16_t*>(codes + d) = static_cast<uint16_t>(c2);
  }
  return sc;
}

// Two E4M3 codes -> a bf16 pair (exact: every E4M3 value is a bf16 value).
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t c2) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(c2), __NV_E4M3);
  const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
  return pack_bf16(f.x, f.y);
}

// Two E4M3 codes -> an f16 pair (exact: E4M3's range and precision lie
// inside f16's normal and subnormal values), one conversion instruction.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t c2) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(c2), __NV_E4M3);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// A page index of the table, or -1 (reported) when it is outside the pool.
__device__ __forceinline__ int64_t page_of(const DecParams& p, const Dec8Params& q8, int s,
                                           int64_t b) {
  const int64_t pg = q8.page_table[static_cast<int64_t>(s) * q8.max_pages + b];
  if (pg < 0 || pg >= q8.n_pages) {
    report(p.status, DEV_ERR_BAD_INDEX, 88, s, static_cast<int>(pg));
    return -1;
  }
  return pg;
}

// Scan (and append): as dec_scan_kernel, over the index-key pages.  Thread t
// of a quad owns d in [t*D/4, (t+1)*D/4) of its two key rows; the codes are
// widened to f16 pairs in registers (one instruction per pair) and each
// key's dot is scaled by the key's scale before the block maximum.  The
// index query enters the f16 MMA multiplied by a power of two 2^e_r that
// puts its largest magnitude in [2^13, 2^14): every bf16 value within 2^-30
// of that maximum converts to f16 exactly, and the dot is multiplied by
// 2^-e_r afterwards, so the scores are those of the bf16 query.
template <int D_IDX, int BK>
__global__ void __launch_bounds__(256, 4) dec8_scan_kernel(const DecParams p, const Dec8Params q8,
                                                        int nsplit) {
  constexpr int DT = D_IDX / 4;     // codes per thread and key row
  constexpr int NMMA = D_IDX / 16;  // MMAs per 16-key tile
  static_assert(DT % 16 == 0, "a thread's codes are whole 16-byte loads");
  const int s = blockIdx.y;
  const int64_t L = p.seq_len[s];  // written back (L + 1) only by the merge kernel
  if (L < 0 || L / p.B_k >= q8.max_pages) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      p.w.Lcur[s] = -1;
      report(p.status, DEV_ERR_CACHE_FULL, 81, s, static_cast<int>(L));
    }
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (blockIdx.x == 0) {
    // append: the new token quantized into slot L % B_k of its page, warp w
    // taking K and V rows of head w (and warp H_kv the index key)
    const int64_t pg = page_of(p, q8, s, L / p.B_k);
    const int64_t slot = L % p.B_k;
    if (pg >= 0) {
      for (int r = warp; r < p.H_kv; r += 8) {
        const int64_t tok = (pg * p.B_k + slot) * p.H_kv + r;
        const float sk = quantize_row_warp(p.k_new + (static_cast<int64_t>(s) * p.H_kv + r) * p.d_h,
                                           p.d_h, q8.k_pages + tok * p.d_h);
        const float sv = quantize_row_warp(p.v_new + (static_cast<int64_t>(s) * p.H_kv + r) * p.d_h,
                                           p.d_h, q8.v_pages + tok * p.d_h);
        if (lane == 0) {
          q8.k_scale[tok] = sk;
          q8.v_scale[tok] = sv;
        }
      }
      if (warp == 7) {
        const float si = quantize_row_warp(p.k_idx_new + static_cast<int64_t>(s) * D_IDX, D_IDX,
                                           q8.kidx_pages + (pg * p.B_k + slot) * D_IDX);
        if (lane == 0) q8.kidx_scale[pg * p.B_k + slot] = si;
      }
    }
    if (threadIdx.x == 0) p.w.Lcur[s] = static_cast<int32_t>(L);
  }
  const int64_t b_i = L / p.B_k;  // candidate blocks 0 .. b_i-1 (full, not the local one)
  const int g = lane >> 2, t = lane & 3;
  uint32_t bq[NMMA][2];
  float unscale0, unscale1;  // 2^-e of the heads in columns 2t and 2t+1
  {
    const __nv_bfloat16* qr = p.q_idx + (static_cast<int64_t>(s) * p.H_kv + (g < p.H_kv ? g : 0)) * D_IDX;
    float qv[NMMA][4];
    float amax = 0.f;
#pragma unroll
    for (int j = 0; j < NMMA; ++j) {
      const int d0 = t * DT + 4 * j;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qv[j][e] = g < p.H_kv ? __bfloat162float(qr[d0 + e]) : 0.f;
        amax = fmaxf(amax, fabsf(qv[j][e]));
      }
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
    const int shift = amax > 0.f ? min(13 - ilogbf(amax), 126) : 0;
#pragma unroll
    for (int j = 0; j < NMMA; ++j) {
      const __half2 lo = __floats2half2_rn(ldexpf(qv[j][0], shift), ldexpf(qv[j][1], shift));
      const __half2 hi = __floats2half2_rn(ldexpf(qv[j][2], shift), ldexpf(qv[j][3], shift));
      bq[j][0] = *reinterpret_cast<const uint32_t*>(&lo);
      bq[j][1] = *reinterpret_cast<const uint32_t*>(&hi);
    }
    unscale0 = ldexpf(1.f, -__shfl_sync(0xFFFFFFFFu, shift, (2 * t) * 4));
    unscale1 = ldexpf(1.f, -__shfl_sync(0xFFFFFFFFu, shift, (2 * t + 1) * 4));
  }
  const int wstride = nsplit * 8;
  // the next block's page index is fetched while this block's codes load
  const int* ptab = q8.page_table + static_cast<int64_t>(s) * q8.max_pages;
  int pg_next = blockIdx.x * 8 + warp < b_i ? __ldg(ptab + blockIdx.x * 8 + warp) : 0;
  for (int64_t b = blockIdx.x * 8 + warp; b < b_i; b += wstride) {
    const int64_t pg = pg_next;
    if (b + wstride < b_i) pg_next = __ldg(ptab + b + wstride);
    if (pg < 0 || pg >= q8.n_pages) {
      report(p.status, DEV_ERR_BAD_INDEX, 88, s, static_cast<int>(pg));
      continue;
    }
    const uint8_t* kbase = q8.kidx_pages + pg * BK * D_IDX;
    const float* sbase = q8.kidx_scale + pg * BK;
    float mx0 = -INFINITY, mx1 = -INFINITY;  // columns 2t, 2t+1
    // the block in two halves of NTILE/2 tiles: each half's codes are all
    // loaded before its arithmetic, so they are in flight together
    constexpr int NTILE = BK / 16, NU = DT / 16, HALF = NTILE / 2;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint4 cr0[HALF][NU], cr1[HALF][NU];
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const uint8_t* r0 = kbase + ((h * HALF + i) * 16 + g) * D_IDX + t * DT;
        const uint8_t* r1 = r0 + 8 * D_IDX;
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          cr0[i][u] = __ldg(reinterpret_cast<const uint4*>(r0) + u);
          cr1[i][u] = __ldg(reinterpret_cast<const uint4*>(r1) + u);
        }
      }
#pragma unroll
      for (int i = 0; i < HALF; ++i) {
        const int tile = h * HALF + i;
        uint32_t w0[DT / 2], w1[DT / 2];  // f16 pairs of rows g and g + 8
#pragma unroll
        for (int u = 0; u < NU; ++u) {
          const uint16_t* h0 = reinterpret_cast<const uint16_t*>(&cr0[i][u]);
          const uint16_t* h1 = reinterpret_cast<const uint16_t*>(&cr1[i][u]);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            w0[u * 8 + e] = e4m3x2_to_f16x2(h0[e]);
            w1[u * 8 + e] = e4m3x2_to_f16x2(h1[e]);
          }
        }
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < NMMA; ++j) {
          // k-slots 2t,2t+1 <- d0,d0+1 ; 2t+8,2t+9 <- d0+2,d0+3 (d0 = t*DT + 4j)
          const uint32_t a[4] = {w0[2 * j], w1[2 * j], w0[2 * j + 1], w1[2 * j + 1]};
          mma_f16_16816(c, a, bq[j][0], bq[j][1]);
        }
        const float s0 = __ldg(sbase + tile * 16 + g), s1 = __ldg(sbase + tile * 16 + g + 8);
        mx0 = fmax3(mx0, (c[0] * unscale0) * s0, (c[2] * unscale0) * s1);
        mx1 = fmax3(mx1, (c[1] * unscale1) * s0, (c[3] * unscale1) * s1);
      }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, o));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, o));
    }
    if (g == 0) {
      const int r0 = 2 * t, r1 = 2 * t + 1;
      float* Mrow = p.w.M + static_cast<int64_t>(s) * p.H_kv * p.Bmax;
      if (r0 < p.H_kv) Mrow[r0 * p.Bmax + b] = mx0;
      if (r1 < p.H_kv) Mrow[r1 * p.Bmax + b] = mx1;
    }
  }
}

// Shared memory of the FP8 attend: one bf16 tile (K, then V over it) that
// later also holds the warps' O rows for their merge.
template <int D_H, int BK>
struct Attend8Smem {
  static constexpr int TILE = BK * D_H * 2;
  static constexpr int OBUF = 4 * 16 * D_H * 4;
  static constexpr int REGION = TILE > OBUF ? TILE : OBUF;
};

// Gathered attention: as dec_attend_kernel, with the selected page's K and V
// codes of head r widened to bf16 into the swizzled tile layout by all
// threads (plain loads: a key's d_h codes are one contiguous row), the keys'
// scales staged in shared memory, S scaled per key and P per value.  K and V
// share one tile: the V codes wait in registers (all loads are issued at the
// start) and are widened over K once every warp has computed S, which halves
// the shared memory of a CTA so that more CTAs (items) run on an SM at once.
template <int D_H, int BK>
__global__ void __launch_bounds__(128) dec8_attend_kernel(const DecParams p, const Dec8Params q8) {
  griddep_wait();  // the previous kernel of the step has finished
  using SM = Attend8Smem<D_H, BK>;
  constexpr int KW = BK / 4;          // keys per warp
  constexpr int NT = KW / 8;          // S n-tiles per warp
  constexpr int DT = D_H / 8;         // O n-tiles
  constexpr int CPK = D_H / 16;       // 16-code pieces per key row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sT = smem;                                          // K tile, then V tile
  float* red = reinterpret_cast<float*>(smem + SM::REGION);  // [4][16] m, [4][16] l
  float* ksc = red + 128;                                    // [BK] key scales
  float* vsc = ksc + BK;                                     // [BK] value scales
  float* obuf = reinterpret_cast<float*>(smem);  // [4][16][D_H], over the V tile once it is used

  const int item = blockIdx.x;  // (s, r, slot)
  const int slot = item % p.kk;
  const int r = (item / p.kk) % p.H_kv;
  const int s = item / (p.kk * p.H_kv);
  // both loads issue before either is tested (they do not depend on each other)
  const int64_t L = p.w.Lcur[s];
  const int b = p.w.sel[(static_cast<int64_t>(s) * p.H_kv + r) * p.kk + slot];
  if (L < 0 || b < 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  // Q fragments (rows = heads, zero beyond G), in flight with the page lookup
  uint32_t qa[D_H / 16][4];
  {
    const __nv_bfloat16* qb = p.q + (static_cast<int64_t>(s) * p.H_q + r * p.G) * D_H;
#pragma unroll
    for (int ks = 0; ks < D_H / 16; ++ks) {
      const int d = ks * 16 + 2 * t;
      qa[ks][0] = g < p.G ? *reinterpret_cast<const uint32_t*>(qb + g * D_H + d) : 0u;
      qa[ks][1] = g + 8 < p.G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D_H + d) : 0u;
      qa[ks][2] = g < p.G ? *reinterpret_cast<const uint32_t*>(qb + g * D_H + d + 8) : 0u;
      qa[ks][3] = g + 8 < p.G ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D_H + d + 8) : 0u;
    }
  }
  const int64_t pg = page_of(p, q8, s, b);
  if (pg < 0) return;
  const int64_t last = L;  // the new token's position: keys j <= last

  // the block's codes -> bf16 tiles [d-chunk][key][64] with 128-byte swizzle;
  // every load of the thread is issued before the first conversion, so the
  // CTA has its whole 2*BK*D_H bytes in flight at once
  constexpr int PER_T = BK * CPK / 128;  // 16-code pieces per thread and tensor
  static_assert(BK * CPK % 128 == 0, "pieces divide over the 128 threads");
  uint4 kcs[PER_T], vcs[PER_T];
#pragma unroll
  for (int i = 0; i < PER_T; ++i) {
    const int c = threadIdx.x + i * 128;
    const int key = c / CPK, piece = c - key * CPK;
    const int64_t row = ((pg * BK + key) * p.H_kv + r) * D_H + piece * 16;
    kcs[i] = __ldg(reinterpret_cast<const uint4*>(q8.k_pages + row));
    vcs[i] = __ldg(reinterpret_cast<const uint4*>(q8.v_pages + row));
  }
  float ks_reg = 0.f, vs_reg = 0.f;
  if (threadIdx.x < BK) {
    ks_reg = __ldg(q8.k_scale + (pg * BK + threadIdx.x) * p.H_kv + r);
    vs_reg = __ldg(q8.v_scale + (pg * BK + threadIdx.x) * p.H_kv + r);
  }
  // 16-code pieces -> bf16 pieces of the swizzled tile
  auto widen = [&](const uint4 (&codes)[PER_T]) {
#pragma unroll
    for (int i = 0; i < PER_T; ++i) {
      const int c = threadIdx.x + i * 128;
      const int key = c / CPK, piece = c - key * CPK;
      const uint16_t* h = reinterpret_cast<const uint16_t*>(&codes[i]);
      uint4 x0, x1;
      uint32_t* p0 = reinterpret_cast<uint32_t*>(&x0);
      uint32_t* p1 = reinterpret_cast<uint32_t*>(&x1);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        p0[e] = e4m3x2_to_bf16x2(h[e]);
        p1[e] = e4m3x2_to_bf16x2(h[4 + e]);
      }
      const int d = piece * 16;
      *reinterpret_cast<uint4*>(sT + sw_addr<BK>(0u, key, d)) = x0;
      *reinterpret_cast<uint4*>(sT + sw_addr<BK>(0u, key, d + 8)) = x1;
    }
  };
  widen(kcs);
  static_assert(BK <= 128, "one key scale per thread");
  if (threadIdx.x < BK) {
    ksc[threadIdx.x] = ks_reg;
    vsc[threadIdx.x] = vs_reg;
  }
  __syncthreads();
  const int kw0 = warp * KW;  // first key (within the block) of this warp
  float sacc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) sacc[n][0] = sacc[n][1] = sacc[n][2] = sacc[n][3] = 0.f;
  {
    const uint32_t kb = smem_u32(sT);
#pragma unroll
    for (int ks = 0; ks < D_H / 16; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < NT / 2; ++n2) {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kw0 + n2 * 16 + (mi >> 1) * 8 + rr;
        const int d = ks * 16 + (mi & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sw_addr<BK>(kb, key, d), b0, b1, b2, b3);
        mma_bf16_16816(sacc[2 * n2], qa[ks], b0, b1);
        mma_bf16_16816(sacc[2 * n2 + 1], qa[ks], b2, b3);
      }
    }
  }
  // key scale, softmax scale, causal mask (the block holding the new token)
  const int64_t j0 = static_cast<int64_t>(b) * BK + kw0;
  float m_lo = -INFINITY, m_hi = -INFINITY;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int kl = kw0 + n * 8 + 2 * t + (e & 1);
      const int64_t j = j0 + n * 8 + 2 * t + (e & 1);
      float x = sacc[n][e] * ksc[kl] * p.scale_log2;
      if (j > last) x = -INFINITY;
      sacc[n][e] = x;
    }
    m_lo = fmax3(m_lo, sacc[n][0], sacc[n][1]);
    m_hi = fmax3(m_hi, sacc[n][2], sacc[n][3]);
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    m_lo = fmaxf(m_lo, __shfl_xor_sync(0xFFFFFFFFu, m_lo, o));
    m_hi = fmaxf(m_hi, __shfl_xor_sync(0xFFFFFFFFu, m_hi, o));
  }
  const float ms_lo = m_lo == -INFINITY ? 0.f : m_lo;
  const float ms_hi = m_hi == -INFINITY ? 0.f : m_hi;
  float l_lo = 0.f, l_hi = 0.f;
  uint32_t pa[NT / 2][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    const float e0 = exp2f(sacc[n][0] - ms_lo), e1 = exp2f(sacc[n][1] - ms_lo);
    const float e2 = exp2f(sacc[n][2] - ms_hi), e3 = exp2f(sacc[n][3] - ms_hi);
    l_lo += e0 + e1;
    l_hi += e2 + e3;
    // the weights times the values' scales, so P V runs on the raw codes
    const int kl = kw0 + n * 8 + 2 * t;
    const float v0 = vsc[kl], v1 = vsc[kl + 1];
    pa[n >> 1][(n & 1) * 2 + 0] = pack_bf16(e0 * v0, e1 * v1);
    pa[n >> 1][(n & 1) * 2 + 1] = pack_bf16(e2 * v0, e3 * v1);
  }
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    l_lo += __shfl_xor_sync(0xFFFFFFFFu, l_lo, o);
    l_hi += __shfl_xor_sync(0xFFFFFFFFu, l_hi, o);
  }
  __syncthreads();  // every warp has read K
  widen(vcs);
  __syncthreads();
  float oacc[DT][4];
#pragma unroll
  for (int n = 0; n < DT; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  {
    const uint32_t vb = smem_u32(sT);
#pragma unroll
    for (int ks = 0; ks < NT / 2; ++ks) {
#pragma unroll
      for (int n2 = 0; n2 < DT / 2; ++n2) {
        const int mi = lane >> 3, rr = lane & 7;
        const int key = kw0 + ks * 16 + (mi & 1) * 8 + rr;
        const int d = n2 * 16 + (mi >> 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(sw_addr<BK>(vb, key, d), b0, b1, b2, b3);
        mma_bf16_16816(oacc[2 * n2], pa[ks], b0, b1);
        mma_bf16_16816(oacc[2 * n2 + 1], pa[ks], b2, b3);
      }
    }
  }
  // merge the four warps' (m, l, O) through shared memory, as dec_attend_kernel
  __syncthreads();
  if (t == 0) {
    red[warp * 16 + g] = m_lo;
    red[warp * 16 + g + 8] = m_hi;
    red[64 + warp * 16 + g] = l_lo;
    red[64 + warp * 16 + g + 8] = l_hi;
  }
#pragma unroll
  for (int n = 0; n < DT; ++n) {
    float* o0 = obuf + (warp * 16 + g) * D_H + n * 8 + 2 * t;
    float* o1 = obuf + (warp * 16 + g + 8) * D_H + n * 8 + 2 * t;
    o0[0] = oacc[n][0];
    o0[1] = oacc[n][1];
    o1[0] = oacc[n][2];
    o1[1] = oacc[n][3];
  }
  __syncthreads();
  const int hr = threadIdx.x >> 3, part = threadIdx.x & 7;
  if (hr < p.G) {
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red[w * 16 + hr]);
    const float Ms = M == -INFINITY ? 0.f : M;
    float wsum = 0.f, wt[4];
    for (int w = 0; w < 4; ++w) {
      const float mw = red[w * 16 + hr];
      wt[w] = mw == -INFINITY ? 0.f : exp2f(mw - Ms);
      wsum += wt[w] * red[64 + w * 16 + hr];
    }
    const int64_t pslot = ((static_cast<int64_t>(s) * p.H_kv + r) * p.kk + slot) * p.G + hr;
    float* dst = p.w.part_o + pslot * D_H;
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    for (int d = part; d < D_H; d += 8) {
      float acc = 0.f;
      for (int w = 0; w < 4; ++w) acc += wt[w] * obuf[(w * 16 + hr) * D_H + d];
      dst[d] = acc * inv;
    }
    if (part == 0)
      p.w.part_lse[pslot] = wsum > 0.f ? (M + log2f(wsum)) * 0.6931471805599453f : -INFINITY;
  }
}

// CTAs per sequence of the FP8 scan: the S sequences share one wave of the
// CTAs the device holds at once (resident CTAs per SM from the kernel's
// registers, times the SMs), at most 64.
template <int D_IDX, int BK>
int scan8_split(int S) {
  static std::atomic<int> slots{0};
  int n = slots.load(std::memory_order_relaxed);
  if (n == 0) {
    int dev = 0, sms = 0, occ = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, dec8_scan_kernel<D_IDX, BK>, 256, 0);
    n = (occ > 0 ? occ : 1) * (sms > 0 ? sms : 1);
    slots.store(n, std::memory_order_relaxed);
  }
  const int per = n / (S > 0 ? S : 1);
  return per < 1 ? 1 : (per > 64 ? 64 : per);
}

template <int D_H, int BK>
size_t attend8_smem() {
  return 1024 + Attend8Smem<D_H, BK>::REGION + 128 * 4 + 2 * BK * 4;
}

// Per-row E4M3 quantization of bf16 rows (for filling a cache): one warp per row.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16* x, int64_t n_rows,
                                                            int dim, uint8_t* codes, float* scales) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (row >= n_rows) return;
  const float sc = quantize_row_warp(x + row * dim, dim, codes + row * dim);
  if ((threadIdx.x & 31) == 0) scales[row] = sc;
}

}  // namespace

size_t decode_workspace_bytes(int S, int64_t L_max, int H_q, int H_kv, int d_h, int B_k, int kk) {
  size_t total = 0;
  carve(nullptr, S, L_max, H_q, H_kv, d_h, B_k, kk, &total);
  return total;
}

cudaError_t launch_decode(const DecodeLaunch& a, cudaStream_t stream) {
  DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.q_idx = static_cast<const __nv_bfloat16*>(a.q_idx);
  p.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(a.v_new);
  p.k_idx_new = static_cast<const __nv_bfloat16*>(a.k_idx_new);
  p.k_cache = static_cast<__nv_bfloat16*>(a.k_cache);
  p.v_cache = static_cast<__nv_bfloat16*>(a.v_cache);
  p.k_idx_cache = static_cast<__nv_bfloat16*>(a.k_idx_cache);
  p.seq_len = a.seq_len;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.idx_out = a.idx_out;
  p.S = a.S;
  p.L_max = a.L_max;
  p.Bmax = (a.L_max + a.B_k - 1) / a.B_k + 1;
  p.H_q = a.H_q;
  p.H_kv = a.H_kv;
  p.d_h = a.d_h;
  p.d_idx = a.d_idx;
  p.B_k = a.B_k;
  p.kk = a.kk;
  p.G = a.H_q / a.H_kv;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  size_t need = 0;
  p.w = carve(a.ws, a.S, a.L_max, a.H_q, a.H_kv, a.d_h, a.B_k, a.kk, &need);
  if (need > a.ws_bytes) return cudaErrorInvalidValue;
  p.status = a.status;

  cudaError_t e = cudaSuccess;
  switch (a.d_idx) {
    case 32: e = launch_scan<32>(p, stream); break;
    case 64: e = launch_scan<64>(p, stream); break;
    case 128: e = launch_scan<128>(p, stream); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int hs = a.kk - 1 > 0 ? a.kk - 1 : 1;
  const size_t topk_smem = (8 * hs * 32 + 8 * hs) * sizeof(uint64_t);
  e = cudaFuncSetAttribute(dec_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(topk_smem));
  if (e != cudaSuccess) return e;
  prof_begin("dec_topk", stream);
  e = launch_pdl(dec_topk_kernel, dim3(a.S * a.H_kv), dim3(256), topk_smem, stream, p);
  prof_end(stream);
  if (e != cudaSuccess) return e;
  if (a.d_h == 128 && a.B_k == 128) e = launch_attend<128, 128>(p, stream);
  else if (a.d_h == 128 && a.B_k == 64) e = launch_attend<128, 64>(p, stream);
  else if (a.d_h == 64 && a.B_k == 128) e = launch_attend<64, 128>(p, stream);
  else e = launch_attend<64, 64>(p, stream);
  if (e != cudaSuccess) return e;
  const int rows = a.S * a.H_q;
  prof_begin("dec_merge", stream);
  e = launch_pdl(a.d_h == 128 ? dec_merge_kernel<128> : dec_merge_kernel<64>,
                 dim3((rows * 32 + 255) / 256), dim3(256), 0, stream, p);
  prof_end(stream);
  return e != cudaSuccess ? e : cudaGetLastError();
}

size_t paged_decode_workspace_bytes(int S, int max_pages, int H_q, int H_kv, int d_h, int B_k,
                                    int kk) {
  return decode_workspace_bytes(S, static_cast<int64_t>(max_pages) * B_k, H_q, H_kv, d_h, B_k, kk);
}

cudaError_t launch_paged_decode_fp8(const PagedLaunch& a, cudaStream_t stream) {
  DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.q_idx = static_cast<const __nv_bfloat16*>(a.q_idx);
  p.k_new = static_cast<const __nv_bfloat16*>(a.k_new);
  p.v_new = static_cast<const __nv_bfloat16*>(a.v_new);
  p.k_idx_new = static_cast<const __nv_bfloat16*>(a.k_idx_new);
  p.k_cache = nullptr;
  p.v_cache = nullptr;
  p.k_idx_cache = nullptr;
  p.seq_len = a.seq_len;
  p.o = static_cast<__nv_bfloat16*>(a.o);
  p.idx_out = a.idx_out;
  p.S = a.S;
  p.L_max = static_cast<int64_t>(a.max_pages) * a.B_k;
  p.Bmax = a.max_pages + 1;
  p.H_q = a.H_q;
  p.H_kv = a.H_kv;
  p.d_h = a.d_h;
  p.d_idx = a.d_idx;
  p.B_k = a.B_k;
  p.kk = a.kk;
  p.G = a.H_q / a.H_kv;
  p.scale = a.scale;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  size_t need = 0;
  p.w = carve(a.ws, a.S, p.L_max, a.H_q, a.H_kv, a.d_h, a.B_k, a.kk, &need);
  if (need > a.ws_bytes) return cudaErrorInvalidValue;
  p.status = a.status;
  Dec8Params q8;
  q8.k_pages = static_cast<uint8_t*>(a.k_pages);
  q8.k_scale = a.k_scale;
  q8.v_pages = static_cast<uint8_t*>(a.v_pages);
  q8.v_scale = a.v_scale;
  q8.kidx_pages = static_cast<uint8_t*>(a.kidx_pages);
  q8.kidx_scale = a.kidx_scale;
  q8.page_table = a.page_table;
  q8.max_pages = a.max_pages;
  q8.n_pages = a.n_pages;

  int nsplit;
  if (a.d_idx == 64 && a.B_k == 128) nsplit = scan8_split<64, 128>(a.S);
  else if (a.d_idx == 64) nsplit = scan8_split<64, 64>(a.S);
  else if (a.B_k == 128) nsplit = scan8_split<128, 128>(a.S);
  else nsplit = scan8_split<128, 64>(a.S);
  const dim3 sgrid(nsplit, a.S);
  prof_begin("dec8_scan", stream);
  if (a.d_idx == 64 && a.B_k == 128) dec8_scan_kernel<64, 128><<<sgrid, 256, 0, stream>>>(p, q8, nsplit);
  else if (a.d_idx == 64) dec8_scan_kernel<64, 64><<<sgrid, 256, 0, stream>>>(p, q8, nsplit);
  else if (a.B_k == 128) dec8_scan_kernel<128, 128><<<sgrid, 256, 0, stream>>>(p, q8, nsplit);
  else dec8_scan_kernel<128, 64><<<sgrid, 256, 0, stream>>>(p, q8, nsplit);
  prof_end(stream);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int hs = a.kk - 1 > 0 ? a.kk - 1 : 1;
  const size_t topk_smem = (8 * hs * 32 + 8 * hs) * sizeof(uint64_t);
  e = cudaFuncSetAttribute(dec_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(topk_smem));
  if (e != cudaSuccess) return e;
  prof_begin("dec_topk", stream);
  e = launch_pdl(dec_topk_kernel, dim3(a.S * a.H_kv), dim3(256), topk_smem, stream, p);
  prof_end(stream);
  if (e != cudaSuccess) return e;
  auto attend = [&](auto kern, size_t smem) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (r != cudaSuccess) return r;
    prof_begin("dec8_attend", stream);
    r = launch_pdl(kern, dim3(a.S * a.H_kv * a.kk), dim3(128), smem, stream, p, q8);
    prof_end(stream);
    return r != cudaSuccess ? r : cudaGetLastError();
  };
  if (a.d_h == 128 && a.B_k == 128) e = attend(dec8_attend_kernel<128, 128>, attend8_smem<128, 128>());
  else if (a.d_h == 128) e = attend(dec8_attend_kernel<128, 64>, attend8_smem<128, 64>());
  else if (a.B_k == 128) e = attend(dec8_attend_kernel<64, 128>, attend8_smem<64, 128>());
  else e = attend(dec8_attend_kernel<64, 64>, attend8_smem<64, 64>());
  if (e != cudaSuccess) return e;
  const int rows = a.S * a.H_q;
  prof_begin("dec_merge", stream);
  e = launch_pdl(a.d_h == 128 ? dec_merge_kernel<128> : dec_merge_kernel<64>,
                 dim3((rows * 32 + 255) / 256), dim3(256), 0, stream, p);
  prof_end(stream);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quantize_fp8_rows(const void* x, int64_t n_rows, int dim, void* codes,
                                     float* scales, cudaStream_t stream) {
  const int64_t threads = n_rows * 32;
  prof_begin("quantize_fp8_rows", stream);
  quantize_rows_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), n_rows, dim, static_cast<uint8_t*>(codes), scales);
  prof_end(stream);
  return cudaGetLastError();
}

}  // namespace msa

// ------------------------------------------------------------------------
// Decode without a caller workspace (msa_sparse_decode_noalloc in msa.h).
// Callers that cannot allocate device memory while serving get the step's
// scratch from this fixed array instead; every GPU that runs the library's
// kernels holds it until the process exits.
// ------------------------------------------------------------------------
#include "../../include/msa.h"

// Dims-only validation of the decode entry points (msa_capi.cu).
msa_status msa_check_decode_dims(const msa_decode_dims* d);

static __device__ __align__(256) uint8_t g_decode_scratch[MSA_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_decode_scratch in the current device's context.  In
// host code the array's name is only a host-side stand-in, never a usable
// device pointer, so the address is looked up with the device current.  It
// is looked up on every call (cheap once the module is loaded) rather than
// cached per device ordinal: after a cudaDeviceReset, or under another
// context on the same ordinal, the module is loaded anew and an address kept
// from before would point at freed memory.
void* decode_scratch(msa_status* st) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || p == nullptr) {
    *st = MSA_ERR_CUDA;
    return nullptr;
  }
  *st = MSA_OK;
  return p;
}
}  // namespace

extern "C" msa_status msa_sparse_decode_noalloc(const msa_decode_dims* d, const void* q,
                                                const void* q_idx, const void* k_new,
                                                const void* v_new, const void* k_idx_new,
                                                void* k_cache, void* v_cache, void* k_idx_cache,
                                                int32_t* seq_len, void* o, int32_t* idx_out,
                                                void* stream) {
  msa::NvtxRange nvtx_range("msa_sparse_decode_noalloc");
  // the dims are checked before the scratch size is computed from them
  const msa_status dims_ok = msa_check_decode_dims(d);
  if (dims_ok != MSA_OK) return dims_ok;
  const size_t need = msa_sparse_decode_workspace(d);
  if (need == 0) return MSA_ERR_INVALID_ARG;
  if (need > MSA_DECODE_NOALLOC_SCRATCH_BYTES) return MSA_ERR_WORKSPACE_TOO_SMALL;
  msa_status st = MSA_OK;
  void* ws = decode_scratch(&st);
  if (ws == nullptr) return st;
  // The regular entry point validates every argument, clears the status word
  // at the head of the scratch and launches the same kernels.
  return msa_sparse_decode(d, q, q_idx, k_new, v_new, k_idx_new, k_cache, v_cache, k_idx_cache,
                           seq_len, o, idx_out, ws, MSA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}
