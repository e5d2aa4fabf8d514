// index_lse.cu -- the KL-loss fusion's Index Branch normaliser LSE_idx
// (xllm-io review, Eq. 9 and "4.3 Sparse KL Loss Fusion"; chlience notes
// 5.4): the inverse index in 16-slot tiles, each selected block's
// index-score LSE per slot (mma.sync), and a log-sum-exp over a row's slots.
#include "attn_common.cuh"

namespace msa {
namespace {

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

}  // namespace msa
