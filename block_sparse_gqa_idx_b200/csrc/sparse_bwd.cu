// sparse_bwd.cu -- the backward of the Main Branch (Eq. 8 with the selection
// fixed) over the forward's inverse index: dQ, dK, dV.
#include "attn_common.cuh"

namespace msa {
namespace {

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
