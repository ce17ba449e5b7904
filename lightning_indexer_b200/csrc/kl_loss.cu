// Indexer KL loss of the dense warm-up stage, with its gradients (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: in the dense
// warm-up, attention stays dense and only the indexer is trained, by minimising the KL
// divergence between the indexer's distribution and the full attention distribution.
//
// Per query row t with visible keys s < vis(t):
//   p[t,s] = (1/Hq) sum_h softmax_s(scale * Q[t,h].K[s,g(h)])    (target, a constant)
//   I[t,s] = indexer score (tcgen05 kernel of dsa_index), q = softmax_s(I)
//   kl[t]  = sum_s p (log p - log q);  loss = mean_t kl[t]
//   g[t,s] = dloss/dI = (q - p) / T
//   x[t,j,s] = q_idx[t,j].k_idx[s],  G[t,j,s] = g w[t,j] [x > 0]
//   dw[t,j] = sum_s g max(0,x),  dq_idx[t,j] = sum_s G k_idx[s],  dk_idx[s] = sum_t,j G q_idx[t,j]
//
// Passes (rows processed in chunks that bound the fp32 score scratch):
//   1. dense LSE          LSE of the dense causal logits for every (t, h)   [tcgen05 for d = 128,
//                         Hq/Hkv = 8 (kl_dense_tc.cu); warp MMA otherwise]
//   per chunk:
//   2. dsa_index          I for the chunk rows                              [tcgen05]
//   3. row_lse_kernel     log-sum-exp of each I row
//   4. kl_target_kernel   p from recomputed dense logits, kl[t], g in place [tcgen05 for d = 128,
//                         Hq/Hkv = 8, Hkv <= 4 (kl_dense_tc.cu); warp MMA otherwise]
//   5. idx_bwd_row_kernel x recomputed per row; dw, dq_idx (row-stationary) [tcgen05 for
//                         H_I = 64, d_I = 128 (kl_dq_tc_kernel); warp MMA otherwise]
//   6. idx_bwd_col_kernel x recomputed per key tile; dk_idx (key-stationary: one CTA per
//                         key tile and block of 1024 rows owns a partial, then the
//                         partials are added in a fixed order: no atomics, deterministic)
//   then dk_idx -> bf16 and loss = mean(kl) (one block, fixed order).
#include "common.cuh"

namespace dsa {

// tiling of the dense-target kernels: warps per CTA, chunks in flight per warp (the one in
// use included), keys per chunk
constexpr int KL_WARPS = 8;
constexpr int KL_STAGES = 3;
constexpr int KL_CHUNK = 16;

__device__ __forceinline__ void ldmatrix_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ int seq_of_row(const int* cu, int batch, long long row) {
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)cu[mid] <= row) lo = mid; else hi = mid;
  }
  return lo;
}

// ------------------------------------------------------------------ 1. dense LSE
// One warp per (row, KV head): streams the row's visible keys (contiguous) in chunks of 16.
// Writes the base-2 LSE log2 sum_s 2^(scale log2(e) Q.K).
template <int D>
__global__ void __launch_bounds__(KL_WARPS * 32)
    dense_lse_kernel(const uint16_t* Q, const uint16_t* K, const int* cu_q, const int* cu_k, int batch,
                     long long rows, int Hq, int Hkv, float scale_log2, float* lse_out) {
  constexpr int SEGS = D / 8;
  constexpr int TILE = KL_CHUNK * D * 2;
  constexpr int MT = D / 16;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const uint32_t my_s = smem_u32(smem + warp * KL_STAGES * TILE);
  const long long task = (long long)blockIdx.x * KL_WARPS + warp;
  const long long row = task / Hkv;
  if (row >= rows) return;
  const int g = (int)(task % Hkv);
  const int G = Hq / Hkv;
  const int b = seq_of_row(cu_q, batch, row);
  const int i = (int)(row - cu_q[b]);
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
  const int kbase = cu_k[b];
  const uint16_t* Kg = K + (size_t)g * D;
  const size_t stride = (size_t)Hkv * D;
  uint32_t qb[MT][2];
  {
    const bool hv = gid < G;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(Q + ((size_t)row * Hq + g * G + (hv ? gid : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      qb[kk][0] = hv ? __ldg(q32 + kk * 8 + tig) : 0u;
      qb[kk][1] = hv ? __ldg(q32 + kk * 8 + 4 + tig) : 0u;
    }
  }
  const int nchunks = (vis + KL_CHUNK - 1) / KL_CHUNK;
  auto issue = [&](int c, int st) {
#pragma unroll
    for (int j = 0; j < KL_CHUNK * SEGS / 32; ++j) {
      const int e = j * 32 + lane;
      const int r = e / SEGS, seg = e % SEGS;
      const int s = c * KL_CHUNK + r;
      const bool valid = s < vis;
      cp_async_16(my_s + st * TILE + tile_off<D>(r, seg), Kg + (valid ? (size_t)(kbase + s) * stride + seg * 8 : 0),
                  valid);
    }
  };
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int st = 0; st < KL_STAGES - 1; ++st) {
    if (st < nchunks) issue(st, st);
    cp_async_commit();
  }
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % KL_STAGES;
    {
      const int cn = c + KL_STAGES - 1;
      if (cn < nchunks) issue(cn, cn % KL_STAGES);
      cp_async_commit();
    }
    cp_async_wait<KL_STAGES - 1>();
    __syncwarp();
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(my_s + st * TILE + tile_off<D>(lane & 15, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
      mma_bf16_16816(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
    }
    const bool v0 = c * KL_CHUNK + gid < vis, v1 = c * KL_CHUNK + gid + 8 < vis;
    const float x00 = v0 ? s[0] * scale_log2 : -INFINITY, x01 = v0 ? s[1] * scale_log2 : -INFINITY;
    const float x10 = v1 ? s[2] * scale_log2 : -INFINITY, x11 = v1 ? s[3] * scale_log2 : -INFINITY;
    float cm0 = fmaxf(x00, x10), cm1 = fmaxf(x01, x11);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, o));
      cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, o));
    }
    const float mn0 = fmaxf(m0, cm0), mn1 = fmaxf(m1, cm1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
    l0 = l0 * exp2f(m0 - mu0) + exp2f(x00 - mu0) + exp2f(x10 - mu0);
    l1 = l1 * exp2f(m1 - mu1) + exp2f(x01 - mu1) + exp2f(x11 - mu1);
    m0 = mn0;
    m1 = mn1;
    __syncwarp();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (lane < 4) {
    const int h0 = 2 * tig, h1 = h0 + 1;
    if (h0 < G) lse_out[row * Hq + g * G + h0] = l0 > 0.f ? m0 + log2f(l0) : -INFINITY;
    if (h1 < G) lse_out[row * Hq + g * G + h1] = l1 > 0.f ? m1 + log2f(l1) : -INFINITY;
  }
}

// ------------------------------------------------------------------ 3. row LSE of I
// With a selection mask (the sparse-adaptation form), only the selected positions count:
// bit s & 31 of mask[((s >> 7) * mask_rows + row) * 4 + ((s >> 5) & 3)].
__device__ __forceinline__ bool kl_selected(const uint32_t* mask, long long mask_rows, long long row, int s) {
  return !mask || ((__ldg(mask + ((long long)(s >> 7) * mask_rows + row) * 4 + ((s >> 5) & 3)) >> (s & 31)) & 1u);
}

__global__ void row_lse_kernel(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                               long long row_begin, float* lseI, const uint32_t* mask, long long mask_rows) {
  __shared__ float red[32];
  const long long row = row_begin + blockIdx.x;
  const int b = seq_of_row(cu_q, batch, row);
  const int i = (int)(row - cu_q[b]);
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
  const float* src = scores + (long long)blockIdx.x * ld;
  float m = -INFINITY;
  for (int s = threadIdx.x; s < vis; s += blockDim.x)
    if (kl_selected(mask, mask_rows, row, s)) m = fmaxf(m, src[s]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = m;
  __syncthreads();
  m = -INFINITY;
  for (int w = 0; w < (int)blockDim.x / 32; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  const float mu = m == -INFINITY ? 0.f : m;
  float sum = 0.f;
  for (int s = threadIdx.x; s < vis; s += blockDim.x)
    if (kl_selected(mask, mask_rows, row, s)) sum += expf(src[s] - mu);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < (int)blockDim.x / 32; ++w) t += red[w];
    lseI[blockIdx.x] = t > 0.f ? mu + logf(t) : -INFINITY;
  }
}

// ------------------------------------------------------------------ 4. target, KL, g
// One block per row, one warp per KV head.  Each warp recomputes its heads' dense logits
// for 16 keys at a time; the head-sum of the softmax weights is combined in shared memory.
template <int D>
__global__ void __launch_bounds__(256)
    kl_target_kernel(const uint16_t* Q, const uint16_t* K, const int* cu_q, const int* cu_k, int batch,
                     long long row_begin, int Hq, int Hkv, float scale_log2, const float* lse_att,
                     const float* lseI, float* scores, long long ld, float inv_T, float* kl_out) {
  constexpr int SEGS = D / 8;
  constexpr int TILE = KL_CHUNK * D * 2;
  constexpr int MT = D / 16;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float psum[8][KL_CHUNK];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const int g = warp;  // blockDim.x == 32 * Hkv
  const uint32_t my_s = smem_u32(smem + warp * KL_STAGES * TILE);
  const long long row = row_begin + blockIdx.x;
  const int G = Hq / Hkv;
  const int b = seq_of_row(cu_q, batch, row);
  const int i = (int)(row - cu_q[b]);
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
  const int kbase = cu_k[b];
  const uint16_t* Kg = K + (size_t)g * D;
  const size_t stride = (size_t)Hkv * D;
  float* Irow = scores + (long long)blockIdx.x * ld;
  const float lI = lseI[blockIdx.x];
  uint32_t qb[MT][2];
  {
    const bool hv = gid < G;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(Q + ((size_t)row * Hq + g * G + (hv ? gid : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      qb[kk][0] = hv ? __ldg(q32 + kk * 8 + tig) : 0u;
      qb[kk][1] = hv ? __ldg(q32 + kk * 8 + 4 + tig) : 0u;
    }
  }
  const int h0 = 2 * tig, h1 = h0 + 1;
  const float L0 = h0 < G ? lse_att[row * Hq + g * G + h0] : -INFINITY;
  const float L1 = h1 < G ? lse_att[row * Hq + g * G + h1] : -INFINITY;
  const int nchunks = (vis + KL_CHUNK - 1) / KL_CHUNK;
  auto issue = [&](int c, int st) {
#pragma unroll
    for (int j = 0; j < KL_CHUNK * SEGS / 32; ++j) {
      const int e = j * 32 + lane;
      const int r = e / SEGS, seg = e % SEGS;
      const int s = c * KL_CHUNK + r;
      const bool valid = s < vis;
      cp_async_16(my_s + st * TILE + tile_off<D>(r, seg), Kg + (valid ? (size_t)(kbase + s) * stride + seg * 8 : 0),
                  valid);
    }
  };
  float kl = 0.f;
#pragma unroll
  for (int st = 0; st < KL_STAGES - 1; ++st) {
    if (st < nchunks) issue(st, st);
    cp_async_commit();
  }
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % KL_STAGES;
    {
      const int cn = c + KL_STAGES - 1;
      if (cn < nchunks) issue(cn, cn % KL_STAGES);
      cp_async_commit();
    }
    cp_async_wait<KL_STAGES - 1>();
    __syncwarp();
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(my_s + st * TILE + tile_off<D>(lane & 15, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
      mma_bf16_16816(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
    }
    // softmax weights of this warp's heads, summed over the heads, per key
    float e0 = (h0 < G ? exp2f(s[0] * scale_log2 - L0) : 0.f) + (h1 < G ? exp2f(s[1] * scale_log2 - L1) : 0.f);
    float e1 = (h0 < G ? exp2f(s[2] * scale_log2 - L0) : 0.f) + (h1 < G ? exp2f(s[3] * scale_log2 - L1) : 0.f);
    e0 += __shfl_xor_sync(0xffffffffu, e0, 1);
    e0 += __shfl_xor_sync(0xffffffffu, e0, 2);
    e1 += __shfl_xor_sync(0xffffffffu, e1, 1);
    e1 += __shfl_xor_sync(0xffffffffu, e1, 2);
    if (tig == 0) {
      psum[g][gid] = e0;
      psum[g][gid + 8] = e1;
    }
    __syncthreads();
    if (warp == 0 && lane < KL_CHUNK) {
      const int sidx = c * KL_CHUNK + lane;
      if (sidx < vis) {
        float pp = 0.f;
        for (int w = 0; w < Hkv; ++w) pp += psum[w][lane];
        pp *= 1.f / (float)Hq;
        const float lq = Irow[sidx] - lI;  // log q
        if (pp > 0.f) kl += pp * (logf(pp) - lq);
        Irow[sidx] = (expf(lq) - pp) * inv_T;  // g = dloss/dI
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if (warp == 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kl += __shfl_xor_sync(0xffffffffu, kl, o);
    if (lane == 0) kl_out[row] = kl;
  }
}

// ------------------------------------------------------------------ 5. row-stationary
// One block per row t, H_I/16 warps (16 indexer heads each).  Key tiles of 64 rows of
// k_idx stream through shared memory.  Per warp and tile:
//   x[16 heads x 64 keys] = q_idx[t] . k_tile^T;  dw += g relu(x);  G = g w [x > 0]
//   dq[16 heads x d_I] += G . k_tile
template <int H_I, int D_I>
__global__ void __launch_bounds__(H_I / 16 * 32)
    idx_bwd_row_kernel(const uint16_t* q_idx, const uint16_t* k_idx, const uint16_t* w, const int* cu_q,
                       const int* cu_k, int batch, long long row_begin, const float* gbuf, long long ld,
                       uint16_t* dq_out, uint16_t* dw_out) {
  constexpr int KT = 64;            // keys per tile
  constexpr int SEGS = D_I / 8;     // 16-byte segments per k_idx row
  constexpr int TILE = KT * D_I * 2;
  constexpr int NW = H_I / 16;
  constexpr int KS = D_I / 16;      // k-steps of x
  constexpr int NTD = D_I / 8;      // n-tiles of dq
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const uint32_t sbase = smem_u32(smem);
  const long long row = row_begin + blockIdx.x;
  const int b = seq_of_row(cu_q, batch, row);
  const int i = (int)(row - cu_q[b]);
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
  const int kbase = cu_k[b];
  const float* grow = gbuf + (long long)blockIdx.x * ld;
  // A fragments of this warp's 16 heads of q_idx[t]: rows gid, gid+8; k pairs 2*tig (+8)
  uint32_t qa[KS][4];
  {
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(q_idx + ((size_t)row * H_I + warp * 16 + gid) * D_I);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(q_idx + ((size_t)row * H_I + warp * 16 + gid + 8) * D_I);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = __ldg(q0 + kk * 8 + tig);
      qa[kk][1] = __ldg(q1 + kk * 8 + tig);
      qa[kk][2] = __ldg(q0 + kk * 8 + 4 + tig);
      qa[kk][3] = __ldg(q1 + kk * 8 + 4 + tig);
    }
  }
  const float wA = bf16_bits_to_f32(w[row * H_I + warp * 16 + gid]);
  const float wB = bf16_bits_to_f32(w[row * H_I + warp * 16 + gid + 8]);
  float dq[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;
  float dwA = 0.f, dwB = 0.f;
  const int ntiles = (vis + KT - 1) / KT;
  auto issue = [&](int tile, int st) {
    for (int e = threadIdx.x; e < KT * SEGS; e += NW * 32) {
      const int r = e / SEGS, seg = e % SEGS;
      const int s = tile * KT + r;
      const bool valid = s < vis;
      const uint32_t dst = sbase + st * TILE + (uint32_t)(r * D_I * 2 + (((seg & ~7) | ((seg ^ r) & 7)) << 4));
      cp_async_16(dst, k_idx + (valid ? (size_t)(kbase + s) * D_I + seg * 8 : 0), valid);
    }
  };
  // byte offset of segment seg of row r in a [KT][D_I] tile (XOR swizzle within 8-segment groups)
  auto off = [&](int r, int seg) -> uint32_t {
    return (uint32_t)(r * D_I * 2 + (((seg & ~7) | ((seg ^ r) & 7)) << 4));
  };
  if (ntiles > 0) issue(0, 0);
  cp_async_commit();
#pragma unroll 1
  for (int tile = 0; tile < ntiles; ++tile) {
    const int st = tile & 1;
    if (tile + 1 < ntiles) issue(tile + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t kt = sbase + st * TILE;
    // x = q . k^T : 8 n-tiles of 8 keys
    float x[KT / 8][4];
#pragma unroll
    for (int nt = 0; nt < KT / 8; ++nt) {
      x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t b0, b1;
        // B[k = d][n = key]: rows = keys nt*8 + (lane&7), segment 2*kk + (lane>>3 & 1)
        ldmatrix_x2(kt + off(nt * 8 + (lane & 7), kk * 2 + ((lane >> 3) & 1)), b0, b1);
        mma_bf16_16816(x[nt], qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3], b0, b1);
      }
    }
    // G = g w [x > 0] (bf16, A layout), dw += g relu(x)
    uint32_t ga[KT / 16][4];
#pragma unroll
    for (int nt = 0; nt < KT / 8; ++nt) {
      const int s0 = tile * KT + nt * 8 + 2 * tig;
      const float g0 = s0 < vis ? grow[s0] : 0.f;
      const float g1 = s0 + 1 < vis ? grow[s0 + 1] : 0.f;
      dwA += g0 * fmaxf(x[nt][0], 0.f) + g1 * fmaxf(x[nt][1], 0.f);
      dwB += g0 * fmaxf(x[nt][2], 0.f) + g1 * fmaxf(x[nt][3], 0.f);
      const uint32_t lo = pack_bf16x2(x[nt][0] > 0.f ? g0 * wA : 0.f, x[nt][1] > 0.f ? g1 * wA : 0.f);
      const uint32_t hi = pack_bf16x2(x[nt][2] > 0.f ? g0 * wB : 0.f, x[nt][3] > 0.f ? g1 * wB : 0.f);
      ga[nt / 2][(nt & 1) * 2 + 0] = lo;
      ga[nt / 2][(nt & 1) * 2 + 1] = hi;
    }
    // dq += G[16 x 64 keys] . k_tile[64 keys x D_I]
#pragma unroll
    for (int ks = 0; ks < KT / 16; ++ks) {
#pragma unroll
      for (int nd = 0; nd < NTD; ++nd) {
        uint32_t b0, b1;
        // B[k = key][n = d]: transposed load of rows keys ks*16 + (lane & 15), segment nd
        ldmatrix_x2_trans(kt + off(ks * 16 + (lane & 15), nd), b0, b1);
        mma_bf16_16816(dq[nd], ga[ks][0], ga[ks][1], ga[ks][2], ga[ks][3], b0, b1);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    dwA += __shfl_xor_sync(0xffffffffu, dwA, o);
    dwB += __shfl_xor_sync(0xffffffffu, dwB, o);
  }
  if (tig == 0) {
    dw_out[row * H_I + warp * 16 + gid] = __bfloat16_as_ushort(__float2bfloat16_rn(dwA));
    dw_out[row * H_I + warp * 16 + gid + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(dwB));
  }
  uint16_t* qrA = dq_out + ((size_t)row * H_I + warp * 16 + gid) * D_I;
  uint16_t* qrB = dq_out + ((size_t)row * H_I + warp * 16 + gid + 8) * D_I;
#pragma unroll
  for (int nd = 0; nd < NTD; ++nd) {
    const uint32_t lo = pack_bf16x2(dq[nd][0], dq[nd][1]);
    const uint32_t hi = pack_bf16x2(dq[nd][2], dq[nd][3]);
    *reinterpret_cast<uint32_t*>(qrA + nd * 8 + 2 * tig) = lo;
    *reinterpret_cast<uint32_t*>(qrB + nd * 8 + 2 * tig) = hi;
  }
}

// ------------------------------------------------------------------ 6. key-stationary
// One block per (sequence, tile of 128 keys, block of KL_COL_ROWS rows of the chunk), 8
// warps of 16 keys.  Streams its rows that see the tile; per row t:
//   x^T[16 keys x H_I] = k_w . q_idx[t]^T;  G^T = g w [x > 0];  dk[16 x d_I] += G^T . q_idx[t]
// and stores its partial dk to dk_part[row block] (plain stores: every (row block, key)
// entry has one writer); dk_reduce_kernel then adds the row blocks in a fixed order.
constexpr int KL_COL_ROWS = 1024;

// rows [qlo, qhi) of the chunk [row_begin, row_end) that see key tile `tile` of sequence b
__device__ __forceinline__ void col_rows(const int* cu_q, const int* cu_k, int b, int tile, long long row_begin,
                                         long long row_end, long long& qlo, long long& qhi) {
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  qlo = max((long long)cu_q[b] + max(tile * 128 - (Lk - Lq), 0), row_begin);
  qhi = min((long long)cu_q[b + 1], row_end);
}

template <int H_I, int D_I>
__global__ void __launch_bounds__(256)
    idx_bwd_col_kernel(const uint16_t* q_idx, const uint16_t* k_idx, const uint16_t* w, const int* cu_q,
                       const int* cu_k, int batch, long long row_begin, long long row_end, const float* gbuf,
                       long long ld, int tiles_per_seq, int row_blocks, float* dk_part, long long part_stride) {
  constexpr int KT = 128;
  constexpr int SEGS = D_I / 8;
  constexpr int QT = H_I * D_I * 2;  // q_idx[t] tile bytes
  constexpr int KS = D_I / 16;
  constexpr int NTH = H_I / 8;       // n-tiles of heads
  constexpr int KSH = H_I / 16;      // k-steps over heads
  constexpr int NTD = D_I / 8;
  extern __shared__ __align__(128) uint8_t smem[];
  float* s_w = reinterpret_cast<float*>(smem + 2 * QT);   // [2][H_I]
  float* s_g = s_w + 2 * H_I;                             // [2][KT]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const uint32_t sbase = smem_u32(smem);
  const int rb = blockIdx.x % row_blocks;
  const int tile = (blockIdx.x / row_blocks) % tiles_per_seq;
  const int b = blockIdx.x / (row_blocks * tiles_per_seq);
  if (b >= batch) return;
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  const int s0 = tile * KT;
  if (s0 >= Lk) return;
  const int kbase = cu_k[b];
  // this block's rows: block rb of the rows of [row_begin, row_end) that see key s0
  long long qlo, qhi;
  col_rows(cu_q, cu_k, b, tile, row_begin, row_end, qlo, qhi);
  qlo += (long long)rb * KL_COL_ROWS;
  qhi = min(qhi, qlo + KL_COL_ROWS);
  if (qlo >= qhi) return;
  float* dk_acc = dk_part + rb * part_stride;
  // A fragments of this warp's 16 keys of k_idx (zero rows past Lk)
  uint32_t ka[KS][4];
  {
    const int kA = s0 + warp * 16 + gid, kB = kA + 8;
    const uint32_t* p0 = reinterpret_cast<const uint32_t*>(k_idx + (size_t)(kbase + min(kA, Lk - 1)) * D_I);
    const uint32_t* p1 = reinterpret_cast<const uint32_t*>(k_idx + (size_t)(kbase + min(kB, Lk - 1)) * D_I);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      ka[kk][0] = kA < Lk ? __ldg(p0 + kk * 8 + tig) : 0u;
      ka[kk][1] = kB < Lk ? __ldg(p1 + kk * 8 + tig) : 0u;
      ka[kk][2] = kA < Lk ? __ldg(p0 + kk * 8 + 4 + tig) : 0u;
      ka[kk][3] = kB < Lk ? __ldg(p1 + kk * 8 + 4 + tig) : 0u;
    }
  }
  auto off = [&](int r, int seg) -> uint32_t {
    return (uint32_t)(r * D_I * 2 + (((seg & ~7) | ((seg ^ r) & 7)) << 4));
  };
  auto issue = [&](long long row, int st) {
    for (int e = threadIdx.x; e < H_I * SEGS; e += 256) {
      const int r = e / SEGS, seg = e % SEGS;
      cp_async_16(sbase + st * QT + off(r, seg), q_idx + ((size_t)row * H_I + r) * D_I + seg * 8, true);
    }
  };
  float dk[NTD][4];
#pragma unroll
  for (int n = 0; n < NTD; ++n) dk[n][0] = dk[n][1] = dk[n][2] = dk[n][3] = 0.f;
  issue(qlo, 0);
  cp_async_commit();
#pragma unroll 1
  for (long long row = qlo; row < qhi; ++row) {
    const int st = (int)((row - qlo) & 1);
    // small per-row vectors: w[t] and g[t, s0 .. s0+KT) (zero beyond the row's visible range)
    const int i = (int)(row - cu_q[b]);
    const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
    for (int e = threadIdx.x; e < H_I; e += 256) s_w[st * H_I + e] = bf16_bits_to_f32(w[row * H_I + e]);
    for (int e = threadIdx.x; e < KT; e += 256)
      s_g[st * KT + e] = (s0 + e < vis) ? gbuf[(row - row_begin) * ld + s0 + e] : 0.f;
    if (row + 1 < qhi) issue(row + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t qt = sbase + st * QT;
    float x[NTH][4];
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        uint32_t b0, b1;
        ldmatrix_x2(qt + off(nt * 8 + (lane & 7), kk * 2 + ((lane >> 3) & 1)), b0, b1);
        mma_bf16_16816(x[nt], ka[kk][0], ka[kk][1], ka[kk][2], ka[kk][3], b0, b1);
      }
    }
    const float gA = s_g[st * KT + warp * 16 + gid], gB = s_g[st * KT + warp * 16 + gid + 8];
    uint32_t ga[KSH][4];
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      const float w0 = s_w[st * H_I + nt * 8 + 2 * tig], w1 = s_w[st * H_I + nt * 8 + 2 * tig + 1];
      const uint32_t lo = pack_bf16x2(x[nt][0] > 0.f ? gA * w0 : 0.f, x[nt][1] > 0.f ? gA * w1 : 0.f);
      const uint32_t hi = pack_bf16x2(x[nt][2] > 0.f ? gB * w0 : 0.f, x[nt][3] > 0.f ? gB * w1 : 0.f);
      ga[nt / 2][(nt & 1) * 2 + 0] = lo;
      ga[nt / 2][(nt & 1) * 2 + 1] = hi;
    }
#pragma unroll
    for (int ks = 0; ks < KSH; ++ks) {
#pragma unroll
      for (int nd = 0; nd < NTD; ++nd) {
        uint32_t b0, b1;
        ldmatrix_x2_trans(qt + off(ks * 16 + (lane & 15), nd), b0, b1);
        mma_bf16_16816(dk[nd], ga[ks][0], ga[ks][1], ga[ks][2], ga[ks][3], b0, b1);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  const int kA = s0 + warp * 16 + gid, kB = kA + 8;
#pragma unroll
  for (int nd = 0; nd < NTD; ++nd) {
    if (kA < Lk)
      *reinterpret_cast<float2*>(dk_acc + (size_t)(kbase + kA) * D_I + nd * 8 + 2 * tig) = make_float2(dk[nd][0], dk[nd][1]);
    if (kB < Lk)
      *reinterpret_cast<float2*>(dk_acc + (size_t)(kbase + kB) * D_I + nd * 8 + 2 * tig) = make_float2(dk[nd][2], dk[nd][3]);
  }
}

// dk_acc[s] += sum over the row blocks that exist for key s's tile (in block order) of
// dk_part[rb][s]: one thread per 4 consecutive values of one key.
template <int D_I>
__global__ void dk_reduce_kernel(const float* dk_part, long long part_stride, const int* cu_q, const int* cu_k,
                                 int batch, long long row_begin, long long row_end, long long Tk, float* dk_acc) {
  const long long e = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= Tk * D_I) return;
  const long long key = e / D_I;
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)cu_k[mid] <= key) lo = mid; else hi = mid;
  }
  const int tile = (int)((key - cu_k[lo]) / 128);
  long long qlo, qhi;
  col_rows(cu_q, cu_k, lo, tile, row_begin, row_end, qlo, qhi);
  if (qlo >= qhi) return;
  const int nrb = (int)((qhi - qlo + KL_COL_ROWS - 1) / KL_COL_ROWS);
  float4 acc = *reinterpret_cast<const float4*>(dk_acc + e);
  for (int rb = 0; rb < nrb; ++rb) {
    const float4 v = *reinterpret_cast<const float4*>(dk_part + rb * part_stride + e);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  *reinterpret_cast<float4*>(dk_acc + e) = acc;
}

// loss = mean of kl over all rows (one block, fixed summation order)
__global__ void mean_kernel(const float* kl, long long n, float* loss) {
  __shared__ double red[32];
  double s = 0.0;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) s += (double)kl[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)blockDim.x / 32; ++w) t += red[w];
    *loss = n > 0 ? (float)(t / (double)n) : 0.f;
  }
}

}  // namespace dsa

namespace dsa_host {

int indexer_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                   int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k,
                   int H_I, int d_I, long long row_begin, long long row_end, float* scores, long long ld,
                   cudaStream_t stream);
int f32_to_bf16_launch(const float* src, void* dst, long long n, cudaStream_t stream);
int kl_lse_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                     long long Tk, int Hq, int Hkv, int max_seqlen_q, float scale_log2, float* lse_out,
                     cudaStream_t s, const uint32_t* mask, float out_scale, float* max_out,
                     const KlUnion* un);
int kl_target_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                        long long Tk, int Hq, int Hkv, long long r0, long long r1, float scale_log2,
                        const float* lse_att, const float* lseI, float* scores, long long ld, float inv_T,
                        float* kl_part, const uint32_t* mask, cudaStream_t s);
int sa_bwd_mask_build(const int* indices, const int* cu_q, const int* cu_k, int batch, long long total_q, int k,
                      int max_seqlen_k, uint32_t* mask, cudaStream_t s);
int kl_parts_sum_launch(const float* kl_part, long long T, float* kl, cudaStream_t s);
int kl_dq_tc_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                    long long total_q, long long total_k, long long r0, long long r1, const float* g, long long ld,
                    void* dq, void* dw, cudaStream_t s);
int kl_dk_tc_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                    int batch, long long total_q, long long total_k, int max_seqlen_k, long long r0, long long r1,
                    const float* g, long long ld, float* dk_part, int* offs, float* dk_acc, cudaStream_t s);
size_t kl_dk_tc_max_items(long long chunk_rows, long long total_k, int batch, int max_seqlen_k);

struct KLWorkspace {
  float* lse_att;  // [T, Hq] base-2 LSE: log2 sum_s 2^(scale log2(e) Q.K)
  float* dk_acc;   // [Tk, d_I]
  float* dk_part;  // partials of dk: tensor-core path [items][128][d_I], else
                   // [ceil(chunk_rows / KL_COL_ROWS), Tk, d_I] per row block
  int* dk_offs;    // tensor-core path: first item of each (sequence, key tile) pair
  float* lseI;     // [chunk_rows]
  float* scores;   // [chunk_rows, ld]
  float* kl_part;  // [T, 4] per-key-quarter partials of kl (tensor-core target path)
  uint32_t* mask;  // sparse-adaptation form: selection bits [ceil(max_seqlen_k / 128), T, 4]
  size_t total;
};

static size_t r256(size_t x) { return (x + 255) / 256 * 256; }

// the tensor-core backward kernels serve H_I = 64, d_I = 128
static bool kl_tc_backward(int H_I, int d_I) { return H_I == 64 && d_I == 128; }

KLWorkspace kl_workspace_layout(void* base, long long T, long long Tk, int max_seqlen_k, int Hq, int H_I, int d_I,
                                long long chunk_rows, int batch, bool sparse = false) {
  KLWorkspace w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  const size_t ld = ((size_t)(max_seqlen_k > 0 ? max_seqlen_k : 1) + 3) / 4 * 4;
  size_t off = 0;
  w.lse_att = reinterpret_cast<float*>(p + off);
  off += r256((size_t)T * Hq * 4);
  w.dk_acc = reinterpret_cast<float*>(p + off);
  off += r256((size_t)Tk * d_I * 4);
  w.dk_part = reinterpret_cast<float*>(p + off);
  if (kl_tc_backward(H_I, d_I))
    off += r256(kl_dk_tc_max_items(chunk_rows, Tk, batch, max_seqlen_k) * 128 * d_I * 4);
  else
    off += r256((size_t)((chunk_rows + dsa::KL_COL_ROWS - 1) / dsa::KL_COL_ROWS) * Tk * d_I * 4);
  w.dk_offs = reinterpret_cast<int*>(p + off);
  off += r256(((size_t)batch * ((max_seqlen_k + 127) / 128) + 1) * 4);
  w.lseI = reinterpret_cast<float*>(p + off);
  off += r256((size_t)chunk_rows * 4);
  w.scores = reinterpret_cast<float*>(p + off);
  off += r256((size_t)chunk_rows * ld * 4);
  w.kl_part = reinterpret_cast<float*>(p + off);
  off += r256((size_t)T * 4 * 4);
  w.mask = reinterpret_cast<uint32_t*>(p + off);
  if (sparse) off += r256((size_t)T * (size_t)((max_seqlen_k + 127) / 128) * 16);
  w.total = off;
  return w;
}

size_t kl_workspace_bytes(long long T, long long Tk, int max_seqlen_k, int Hq, int H_I, int d_I, long long chunk_rows,
                          int batch, bool sparse) {
  return kl_workspace_layout(nullptr, T, Tk, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, sparse).total;
}

template <int H_I, int D_I>
static int kl_backward_kernels(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                               int batch, long long r0, long long r1, long long T, long long Tk, const float* g,
                               long long ld, int max_seqlen_k, void* dq, void* dw, float* dk_acc, float* dk_part,
                               int* dk_offs, cudaStream_t s) {
  if constexpr (H_I == 64 && D_I == 128) {
    // tensor-core row-stationary kernel
    const int st = kl_dq_tc_launch(q_idx, k_idx, w, cu_q, cu_k, batch, T, Tk, r0, r1, g, ld, dq, dw, s);
    if (st != DSA_OK) return st;
  } else {
    auto kern = dsa::idx_bwd_row_kernel<H_I, D_I>;
    const int smem = 2 * 64 * D_I * 2;
    static DeviceFlag done;
    if (!done) {
      if (const cudaError_t e_ = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); e_ != cudaSuccess) return cuda_fail(e_);
      done = true;
    }
    kern<<<(unsigned)(r1 - r0), H_I / 16 * 32, smem, s>>>(
        static_cast<const uint16_t*>(q_idx), static_cast<const uint16_t*>(k_idx), static_cast<const uint16_t*>(w),
        cu_q, cu_k, batch, r0, g, ld, static_cast<uint16_t*>(dq), static_cast<uint16_t*>(dw));
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  }
  if constexpr (H_I == 64 && D_I == 128) {
    // tensor-core key-stationary kernel (adds its partials into dk_acc itself)
    return kl_dk_tc_launch(q_idx, k_idx, w, cu_q, cu_k, batch, T, Tk, max_seqlen_k, r0, r1, g, ld, dk_part, dk_offs,
                           dk_acc, s);
  } else {
    (void)dk_offs;
    const long long part_stride = Tk * D_I;
    auto kern = dsa::idx_bwd_col_kernel<H_I, D_I>;
    const int smem = 2 * H_I * D_I * 2 + 2 * H_I * 4 + 2 * 128 * 4;
    static DeviceFlag done;
    if (!done) {
      if (const cudaError_t e_ = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); e_ != cudaSuccess) return cuda_fail(e_);
      done = true;
    }
    const int tiles = (max_seqlen_k + 127) / 128;
    const int row_blocks = (int)((r1 - r0 + dsa::KL_COL_ROWS - 1) / dsa::KL_COL_ROWS);
    kern<<<(unsigned)((long long)batch * tiles * row_blocks), 256, smem, s>>>(
        static_cast<const uint16_t*>(q_idx), static_cast<const uint16_t*>(k_idx), static_cast<const uint16_t*>(w),
        cu_q, cu_k, batch, r0, r1, g, ld, tiles, row_blocks, dk_part, part_stride);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    const long long quads = Tk * D_I / 4;
    if (quads > 0) {
      dsa::dk_reduce_kernel<D_I><<<(unsigned)((quads + 255) / 256), 256, 0, s>>>(dk_part, part_stride, cu_q, cu_k, batch,
                                                                                 r0, r1, Tk, dk_acc);
      if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    }
  }
  return DSA_OK;
}

// The indexer KL loss.  indices == nullptr: the dense warm-up form over every visible
// position.  Otherwise the sparse-adaptation form over each row's selected set (indices
// [T, k], sequence-local, -1 unused; tensor-core shapes only): the attention LSE, the row
// LSE of I, the target and g all count only the selected positions, and g = 0 elsewhere, so
// the backward kernels are those of the dense form.
int indexer_kl_loss_launch(const void* Q, const void* K, const void* q_idx, const void* k_idx, const void* w,
                           const int* cu_q, const int* cu_k, int batch, long long T, long long Tk,
                           int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d, int H_I, int d_I,
                           float scale, long long chunk_rows, float* loss, float* kl, void* dq, void* dk, void* dw,
                           void* ws, cudaStream_t s, const int* indices, int k) {
  const bool sparse = indices != nullptr;
  KLWorkspace W = kl_workspace_layout(ws, T, Tk, max_seqlen_k, Hq, H_I, d_I, chunk_rows, batch, sparse);
  const long long ld = ((long long)(max_seqlen_k > 0 ? max_seqlen_k : 1) + 3) / 4 * 4;
  const float scale_log2 = scale * 1.4426950408889634f;
  if (const cudaError_t e_ = cudaMemsetAsync(W.dk_acc, 0, (size_t)Tk * d_I * 4, s); e_ != cudaSuccess) return cuda_fail(e_);
  const uint32_t* mask = nullptr;
  if (sparse) {
    if (!(d == 128 && Hq == 8 * Hkv && Hkv <= 4)) return DSA_ERR_UNSUPPORTED;
    const int st = sa_bwd_mask_build(indices, cu_q, cu_k, batch, T, k, max_seqlen_k, W.mask, s);
    if (st != DSA_OK) return st;
    mask = W.mask;
  }
  // 1. attention LSE over the visible (dense) or selected (sparse) positions (tensor cores
  //    for d = 128 and 8 query heads per KV head)
  if (d == 128 && Hq == 8 * Hkv) {
    const int st = kl_lse_tc_launch(Q, K, cu_q, cu_k, batch, T, Tk, Hq, Hkv, max_seqlen_q, scale_log2, W.lse_att, s, mask,
                                    1.f, nullptr, nullptr);
    if (st != DSA_OK) return st;
  } else {
    const long long tasks = T * Hkv;
    const long long blocks = (tasks + dsa::KL_WARPS - 1) / dsa::KL_WARPS;
    const int smem = dsa::KL_WARPS * dsa::KL_STAGES * dsa::KL_CHUNK * d * 2;
    if (blocks > 0) {
      if (d == 128) {
        static DeviceFlag done;
        if (!done) {
          const cudaError_t e_ = cudaFuncSetAttribute(dsa::dense_lse_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          smem);
          if (e_ != cudaSuccess) return cuda_fail(e_);
        }
        done = true;
        dsa::dense_lse_kernel<128><<<(unsigned)blocks, dsa::KL_WARPS * 32, smem, s>>>(
            static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(K), cu_q, cu_k, batch, T, Hq, Hkv,
            scale_log2, W.lse_att);
      } else {
        static DeviceFlag done;
        if (!done) {
          const cudaError_t e_ = cudaFuncSetAttribute(dsa::dense_lse_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          smem);
          if (e_ != cudaSuccess) return cuda_fail(e_);
        }
        done = true;
        dsa::dense_lse_kernel<64><<<(unsigned)blocks, dsa::KL_WARPS * 32, smem, s>>>(
            static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(K), cu_q, cu_k, batch, T, Hq, Hkv,
            scale_log2, W.lse_att);
      }
      if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    }
  }
  const float inv_T = T > 0 ? 1.f / (float)T : 0.f;
  // 4. on tensor cores for d = 128 and 8 query heads per KV head (at most 4 KV heads)
  const bool target_tc = d == 128 && Hq == 8 * Hkv && Hkv <= 4;
  for (long long r0 = 0; r0 < T; r0 += chunk_rows) {
    const long long r1 = std::min(T, r0 + chunk_rows);
    int st = indexer_launch(q_idx, k_idx, w, cu_q, cu_k, batch, T, Tk, max_seqlen_q, max_seqlen_k, H_I, d_I, r0, r1,
                            W.scores, ld, s);
    if (st != DSA_OK) return st;
    dsa::row_lse_kernel<<<(unsigned)(r1 - r0), 256, 0, s>>>(W.scores, ld, cu_q, cu_k, batch, r0, W.lseI, mask, T);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    if (target_tc) {
      st = kl_target_tc_launch(Q, K, cu_q, cu_k, batch, T, Tk, Hq, Hkv, r0, r1, scale_log2, W.lse_att, W.lseI,
                               W.scores, ld, inv_T, W.kl_part, mask, s);
      if (st != DSA_OK) return st;
    } else {
      const int smem = Hkv * dsa::KL_STAGES * dsa::KL_CHUNK * d * 2;
      if (d == 128) {
        static DeviceFlag done;
        if (!done) {
          const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_target_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          8 * dsa::KL_STAGES * dsa::KL_CHUNK * 128 * 2);
          if (e_ != cudaSuccess) return cuda_fail(e_);
        }
        done = true;
        dsa::kl_target_kernel<128><<<(unsigned)(r1 - r0), 32 * Hkv, smem, s>>>(
            static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(K), cu_q, cu_k, batch, r0, Hq, Hkv,
            scale_log2, W.lse_att, W.lseI, W.scores, ld, inv_T, kl);
      } else {
        static DeviceFlag done;
        if (!done) {
          const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_target_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          8 * dsa::KL_STAGES * dsa::KL_CHUNK * 64 * 2);
          if (e_ != cudaSuccess) return cuda_fail(e_);
        }
        done = true;
        dsa::kl_target_kernel<64><<<(unsigned)(r1 - r0), 32 * Hkv, smem, s>>>(
            static_cast<const uint16_t*>(Q), static_cast<const uint16_t*>(K), cu_q, cu_k, batch, r0, Hq, Hkv,
            scale_log2, W.lse_att, W.lseI, W.scores, ld, inv_T, kl);
      }
      if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    }
#define DSA_KLB(HI, DI)                                                                                   \
  if (H_I == HI && d_I == DI) {                                                                          \
    st = kl_backward_kernels<HI, DI>(q_idx, k_idx, w, cu_q, cu_k, batch, r0, r1, T, Tk, W.scores, ld,         \
                                     max_seqlen_k, dq, dw, W.dk_acc, W.dk_part, W.dk_offs, s);               \
    if (st != DSA_OK) return st;                                                                         \
  } else
    DSA_KLB(64, 128) DSA_KLB(32, 128) DSA_KLB(16, 128) { return DSA_ERR_UNSUPPORTED; }
#undef DSA_KLB
  }
  int st = f32_to_bf16_launch(W.dk_acc, dk, Tk * d_I, s);
  if (st != DSA_OK) return st;
  if (target_tc) {
    st = kl_parts_sum_launch(W.kl_part, T, kl, s);
    if (st != DSA_OK) return st;
  }
  dsa::mean_kernel<<<1, 1024, 0, s>>>(kl, T, loss);
  return last_launch_status();
}

}  // namespace dsa_host
