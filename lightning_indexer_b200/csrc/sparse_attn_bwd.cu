// Backward of sparse GQA attention over fixed selected sets (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1, sparse-adaptation
// stage (the whole model trains through sparse attention); QbitAI launch article
// (news.chathome.org): varlen DSA training kernels.
//
// For token t, head h (KV head g), selected key s:
//   P = exp(scale*Q.K - lse),  dP = dO.V,  D = dO.O,  dS = P*(dP - D)
//   dQ[t,h] = scale * sum_s dS K[s,g]          (row-local: registers, written once)
//   dK[s,g] += scale * sum_h dS Q[t,h]         (scatter: fp32 vector reductions)
//   dV[s,g] += sum_h P dO[t,h]
// One warp owns one (token, KV head) and walks its k selected keys in chunks of 16 with
// the same gather ring and swap-AB warp MMAs as the forward kernel.  The head sums of dK
// and dV are MMAs with K = 16 (the 8 heads of the group, zero-padded); their 16 x d
// results go straight to the fp32 workspace with 16-byte reductions (red.global.add.v4.f32,
// after a lane-pair exchange), and a final kernel rounds the workspace to bf16.
#include "common.cuh"

namespace dsa {

// warps per CTA, chunks in flight per warp (the one in use included), keys per chunk
constexpr int BWD_WARPS = 4;
constexpr int BWD_STAGES = 2;
constexpr int BWD_CHUNK = 16;

struct SABwdParams {
  const uint16_t* Q;
  const uint16_t* K;
  const uint16_t* V;
  const uint16_t* O;
  const uint16_t* dO;
  const float* lse;
  const int* indices;
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long rows;
  int Hq, Hkv, G, k;
  float scale, scale_log2;
  uint16_t* dQ;
  float* dK_acc;  // [total_k, Hkv, D] fp32, zeroed before the launch
  float* dV_acc;
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
               : "memory");
}

template <int D>
__global__ void __launch_bounds__(BWD_WARPS * 32, 3) sparse_attn_bwd_kernel(const SABwdParams p) {
  constexpr int SEGS = D / 8;
  constexpr int TILE_BYTES = BWD_CHUNK * D * 2;
  constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int MT = D / 16;  // k-steps over d, and m-tiles of dQ^T
  constexpr int NT = D / 8;   // n-tiles of dK / dV rows
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int gid = lane / 4, tig = lane % 4;
  const uint32_t my_s = smem_u32(smem + warp * BWD_STAGES * STAGE_BYTES);

  // KV head slowest: the resident warps gather from, and reduce into, one head's rows
  const long long task = (long long)blockIdx.x * BWD_WARPS + warp;
  const int g = (int)(task / p.rows);
  if (g >= p.Hkv) return;
  const long long row = task - (long long)g * p.rows;
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)p.cu_q[mid] <= row) lo = mid; else hi = mid;
  }
  const int kbase = p.cu_k[lo];
  const int vis = causal_vis((int)(row - p.cu_q[lo]), p.cu_q[lo + 1] - p.cu_q[lo], p.cu_k[lo + 1] - kbase);
  const int* idx = p.indices + row * p.k;
  const int nchunks = p.k / BWD_CHUNK;
  const size_t kv_row_stride = (size_t)p.Hkv * D;
  const uint16_t* Kg = p.K + (size_t)g * D;
  const uint16_t* Vg = p.V + (size_t)g * D;
  const size_t qoff = ((size_t)row * p.Hq + g * p.G) * D;  // first head of the group

  // B operands over d (S = K.Q^T, dP = V.dO^T): head n = gid, d pairs at 2*tig
  uint32_t qb[MT][2], ob[MT][2];
  // B operands over heads (dK = dS^T.Q, dV = P^T.dO): k = head 2*tig, 2*tig+1; n = d
  uint32_t qh[NT], oh[NT];
  {
    const bool hv = gid < p.G;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(p.Q + qoff + (hv ? gid : 0) * D);
    const uint32_t* o32 = reinterpret_cast<const uint32_t*>(p.dO + qoff + (hv ? gid : 0) * D);
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      qb[kk][0] = hv ? __ldg(q32 + kk * 8 + tig) : 0u;
      qb[kk][1] = hv ? __ldg(q32 + kk * 8 + 4 + tig) : 0u;
      ob[kk][0] = hv ? __ldg(o32 + kk * 8 + tig) : 0u;
      ob[kk][1] = hv ? __ldg(o32 + kk * 8 + 4 + tig) : 0u;
    }
    const int ha = 2 * tig, hb = 2 * tig + 1;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int dd = nt * 8 + gid;
      const uint16_t qa = ha < p.G ? p.Q[qoff + ha * D + dd] : (uint16_t)0;
      const uint16_t qc = hb < p.G ? p.Q[qoff + hb * D + dd] : (uint16_t)0;
      const uint16_t oa = ha < p.G ? p.dO[qoff + ha * D + dd] : (uint16_t)0;
      const uint16_t oc = hb < p.G ? p.dO[qoff + hb * D + dd] : (uint16_t)0;
      qh[nt] = (uint32_t)qa | ((uint32_t)qc << 16);
      oh[nt] = (uint32_t)oa | ((uint32_t)oc << 16);
    }
  }
  // D = dO.O per head (every lane ends with all heads' values), lse in log2 units
  const int h0 = 2 * tig, h1 = h0 + 1;
  float Dh0 = 0.f, Dh1 = 0.f, L0 = -INFINITY, L1 = -INFINITY;
  for (int h = 0; h < p.G; ++h) {
    float part = 0.f;
    for (int dd = lane; dd < D; dd += 32)
      part += bf16_bits_to_f32(p.dO[qoff + h * D + dd]) * bf16_bits_to_f32(p.O[qoff + h * D + dd]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (h == h0) Dh0 = part;
    if (h == h1) Dh1 = part;
  }
  if (h0 < p.G) L0 = p.lse[row * p.Hq + g * p.G + h0] * 1.4426950408889634f;
  if (h1 < p.G) L1 = p.lse[row * p.Hq + g * p.G + h1] * 1.4426950408889634f;
  const bool live0 = L0 > -INFINITY, live1 = L1 > -INFINITY;

  auto issue = [&](int c, int st) {
    const int my_idx = __ldg(idx + c * BWD_CHUNK + (lane & 15));
    const uint32_t kdst = my_s + st * STAGE_BYTES;
    const uint32_t vdst = kdst + TILE_BYTES;
    // eight lanes per row: each copy instruction moves 128-byte pieces (whole lines) of four
    // rows, and a row's slot, validity and address are worked out once for all its pieces
    const int sub = lane >> 3, cc = lane & 7;
#pragma unroll
    for (int j = 0; j < BWD_CHUNK / 4; ++j) {
      const int r = 4 * j + sub;
      const int s = __shfl_sync(0xffffffffu, my_idx, r);
      const bool valid = (unsigned)s < (unsigned)vis;  // -1 and positions the row cannot see
      const size_t off = valid ? (size_t)(kbase + s) * kv_row_stride + cc * 8 : 0;
      const uint32_t o = tile_off<D>(r, cc);
#pragma unroll
      for (int h = 0; h < SEGS / 8; ++h) {  // segment cc + 8h lands 128 h bytes after segment cc
        cp_async_16(kdst + o + h * 128, Kg + off + h * 64, valid);
        cp_async_16(vdst + o + h * 128, Vg + off + h * 64, valid);
      }
    }
  };

  float dq[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) dq[mt][0] = dq[mt][1] = dq[mt][2] = dq[mt][3] = 0.f;

#pragma unroll
  for (int st = 0; st < BWD_STAGES - 1; ++st) {
    if (st < nchunks) issue(st, st);
    cp_async_commit();
  }
#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % BWD_STAGES;
    {
      const int cn = c + BWD_STAGES - 1;
      if (cn < nchunks) issue(cn, cn % BWD_STAGES);
      cp_async_commit();
    }
    cp_async_wait<BWD_STAGES - 1>();
    __syncwarp();
    const uint32_t kt = my_s + st * STAGE_BYTES;
    const uint32_t vt = kt + TILE_BYTES;

    float s[4] = {0.f, 0.f, 0.f, 0.f}, dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4(kt + tile_off<D>(lane & 15, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
      mma_bf16_16816(s, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      ldmatrix_x4(vt + tile_off<D>(lane & 15, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
      mma_bf16_16816(dp, a0, a1, a2, a3, ob[kk][0], ob[kk][1]);
    }
    const int myi = __ldg(idx + c * BWD_CHUNK + (lane & 15));
    const int sA = __shfl_sync(0xffffffffu, myi, gid);      // key of accumulator row gid
    const int sB = __shfl_sync(0xffffffffu, myi, gid + 8);  // key of row gid + 8
    const bool v0 = (unsigned)sA < (unsigned)vis, v1 = (unsigned)sB < (unsigned)vis;
    const float p00 = (v0 && live0) ? exp2f(s[0] * p.scale_log2 - L0) : 0.f;
    const float p01 = (v0 && live1) ? exp2f(s[1] * p.scale_log2 - L1) : 0.f;
    const float p10 = (v1 && live0) ? exp2f(s[2] * p.scale_log2 - L0) : 0.f;
    const float p11 = (v1 && live1) ? exp2f(s[3] * p.scale_log2 - L1) : 0.f;
    const float ds00 = p00 * (dp[0] - Dh0), ds01 = p01 * (dp[1] - Dh1);
    const float ds10 = p10 * (dp[2] - Dh0), ds11 = p11 * (dp[3] - Dh1);
    const uint32_t dsA0 = pack_bf16x2(ds00, ds01), dsA1 = pack_bf16x2(ds10, ds11);
    const uint32_t pA0 = pack_bf16x2(p00, p01), pA1 = pack_bf16x2(p10, p11);

    // dQ^T[d x heads] += K^T[d x 16] . dS^T[16 x heads]
    {
      const uint32_t b0 = movmatrix_trans(dsA0), b1 = movmatrix_trans(dsA1);
      const int vrow = (lane & 7) + ((lane >> 4) << 3);
      const int vseg_off = (lane >> 3) & 1;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(kt + tile_off<D>(vrow, mt * 2 + vseg_off), a0, a1, a2, a3);
        mma_bf16_16816(dq[mt], a0, a1, a2, a3, b0, b1);
      }
    }
    // dK rows = scale * dS^T[16 x heads] . Q_g[heads x d];  dV rows = P^T . dO_g.
    // A lane holds columns (2*tig, 2*tig+1) of rows gid and gid+8; lanes tig and tig^1
    // swap halves so that the even lane owns 4 consecutive columns of row gid and the odd
    // lane the same 4 columns of row gid+8: one 16-byte reduction each.
    const bool odd = tig & 1;
    const bool vmine = odd ? v1 : v0;
    const int smine = odd ? sB : sA;
    float* dkr = p.dK_acc + ((size_t)(kbase + (vmine ? smine : 0)) * p.Hkv + g) * D + 4 * (tig >> 1);
    float* dvr = p.dV_acc + ((size_t)(kbase + (vmine ? smine : 0)) * p.Hkv + g) * D + 4 * (tig >> 1);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float ck[4] = {0.f, 0.f, 0.f, 0.f}, cv[4] = {0.f, 0.f, 0.f, 0.f};
      mma_bf16_16816(ck, dsA0, dsA1, 0u, 0u, qh[nt], 0u);
      mma_bf16_16816(cv, pA0, pA1, 0u, 0u, oh[nt], 0u);
      const float k0 = __shfl_xor_sync(0xffffffffu, odd ? ck[0] : ck[2], 1);
      const float k1 = __shfl_xor_sync(0xffffffffu, odd ? ck[1] : ck[3], 1);
      const float w0 = __shfl_xor_sync(0xffffffffu, odd ? cv[0] : cv[2], 1);
      const float w1 = __shfl_xor_sync(0xffffffffu, odd ? cv[1] : cv[3], 1);
      if (vmine) {
        if (odd) {
          red_add_v4(dkr + nt * 8, k0 * p.scale, k1 * p.scale, ck[2] * p.scale, ck[3] * p.scale);
          red_add_v4(dvr + nt * 8, w0, w1, cv[2], cv[3]);
        } else {
          red_add_v4(dkr + nt * 8, ck[0] * p.scale, ck[1] * p.scale, k0 * p.scale, k1 * p.scale);
          red_add_v4(dvr + nt * 8, cv[0], cv[1], w0, w1);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  uint16_t* dqrow = p.dQ + qoff;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int d0 = mt * 16 + gid;
    if (h0 < p.G) {
      dqrow[h0 * D + d0] = __bfloat16_as_ushort(__float2bfloat16_rn(dq[mt][0] * p.scale));
      dqrow[h0 * D + d0 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(dq[mt][2] * p.scale));
    }
    if (h1 < p.G) {
      dqrow[h1 * D + d0] = __bfloat16_as_ushort(__float2bfloat16_rn(dq[mt][1] * p.scale));
      dqrow[h1 * D + d0 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(dq[mt][3] * p.scale));
    }
  }
}

// fp32 -> bf16 (round to nearest even), 4 elements per thread
__global__ void f32_to_bf16_kernel(const float* __restrict__ src, uint16_t* __restrict__ dst, long long n) {
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 v = *reinterpret_cast<const float4*>(src + i);
    ushort4 o;
    o.x = __bfloat16_as_ushort(__float2bfloat16_rn(v.x));
    o.y = __bfloat16_as_ushort(__float2bfloat16_rn(v.y));
    o.z = __bfloat16_as_ushort(__float2bfloat16_rn(v.z));
    o.w = __bfloat16_as_ushort(__float2bfloat16_rn(v.w));
    *reinterpret_cast<ushort4*>(dst + i) = o;
  } else {
    for (long long j = i; j < n; ++j) dst[j] = __bfloat16_as_ushort(__float2bfloat16_rn(src[j]));
  }
}

}  // namespace dsa

namespace dsa_host {

size_t sparse_attn_bwd_workspace_bytes(long long total_k, int Hkv, int d) {
  return 2 * (((size_t)total_k * Hkv * d * sizeof(float) + 255) / 256 * 256);
}

int f32_to_bf16_launch(const float* src, void* dst, long long n, cudaStream_t stream) {
  if (n <= 0) return DSA_OK;
  const long long threads = (n + 3) / 4;
  const int block = 256;
  const long long grid = (threads + block - 1) / block;
  dsa::f32_to_bf16_kernel<<<(unsigned)grid, block, 0, stream>>>(src, static_cast<uint16_t*>(dst), n);
  return last_launch_status();
}

int sparse_attn_bwd_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                           const float* lse, const int* indices, const int* cu_q, const int* cu_k, int batch,
                           long long total_q, long long total_k, int Hq, int Hkv, int d, int k, float scale,
                           void* dQ, void* dK, void* dV, void* ws, cudaStream_t stream) {
  const size_t half = sparse_attn_bwd_workspace_bytes(total_k, Hkv, d) / 2;
  float* dk_acc = static_cast<float*>(ws);
  float* dv_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + half);
  if (const cudaError_t e_ = cudaMemsetAsync(ws, 0, 2 * half, stream); e_ != cudaSuccess) return cuda_fail(e_);
  dsa::SABwdParams p{};
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.O = static_cast<const uint16_t*>(O);
  p.dO = static_cast<const uint16_t*>(dO);
  p.lse = lse;
  p.indices = indices;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.rows = total_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.k = k;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dQ = static_cast<uint16_t*>(dQ);
  p.dK_acc = dk_acc;
  p.dV_acc = dv_acc;
  const long long tasks = total_q * Hkv;
  const long long blocks = (tasks + dsa::BWD_WARPS - 1) / dsa::BWD_WARPS;
  const int smem = dsa::BWD_WARPS * dsa::BWD_STAGES * 2 * dsa::BWD_CHUNK * d * 2;
  if (blocks > 0) {
    if (d == 128) {
      static DeviceFlag done;
      if (!done) {
        if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sparse_attn_bwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem); e_ != cudaSuccess) return cuda_fail(e_);
        // three CTAs per SM need the largest shared-memory carveout
        if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sparse_attn_bwd_kernel<128>,
                                                        cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            e_ != cudaSuccess) return cuda_fail(e_);
        done = true;
      }
      dsa::sparse_attn_bwd_kernel<128><<<(unsigned)blocks, dsa::BWD_WARPS * 32, smem, stream>>>(p);
    } else {
      static DeviceFlag done;
      if (!done) {
        if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sparse_attn_bwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 smem); e_ != cudaSuccess) return cuda_fail(e_);
        // three CTAs per SM need the largest shared-memory carveout
        if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sparse_attn_bwd_kernel<64>,
                                                        cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            e_ != cudaSuccess) return cuda_fail(e_);
        done = true;
      }
      dsa::sparse_attn_bwd_kernel<64><<<(unsigned)blocks, dsa::BWD_WARPS * 32, smem, stream>>>(p);
    }
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  }
  const long long n = total_k * Hkv * d;
  int st = f32_to_bf16_launch(dk_acc, dK, n, stream);
  if (st != DSA_OK) return st;
  return f32_to_bf16_launch(dv_acc, dV, n, stream);
}

}  // namespace dsa_host
