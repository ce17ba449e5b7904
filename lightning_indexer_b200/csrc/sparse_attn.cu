// Sparse GQA attention over the top-k selected positions (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: attention runs only
// over the positions the indexer selected (O(L*k) instead of O(L^2)), and DSA is adapted
// to GQA: one selected set per token, shared by every query head of that token.
// Section 8 of the same summary: a decode path specific to DSA.
//
// One warp owns one (query row, KV head g, key split).  The G = Hq/Hkv query heads of the
// group share every gathered K/V row.  The work is a gather (k rows of K and V per token
// and group) followed by two tiny products (G x d by d x 16 per 16 keys), so it is bound
// by the gather and by the latency of each warp's dependent chain, not by the tensor
// pipe.  The products use warp-level MMA in swap-AB form (M = 16 keys, N = 8 heads, so no
// M padding is wasted):
//   S^T[16 keys x 8 heads]  = K_chunk[16 x d] . Q_g^T[d x 8]
//   O^T[d x 8 heads]       += V_chunk^T[d x 16] . P^T[16 x 8]
// P^T goes from the accumulator layout to the B-operand layout with movmatrix.trans.
//
// Gather: the K and V rows of a 16-key chunk stream into a per-warp ring of shared-memory
// stages with 16-byte cp.async copies (zero-filling for -1 slots), XOR-swizzled so that
// ldmatrix reads 8 rows without bank conflicts.  The chunk's slot indices are loaded one
// chunk ahead of their copies, so the index load never sits on the issue path.  (Bulk
// 256-byte copies per row, one per lane, were measured slower on B200: the per-copy cost
// of the bulk-copy unit outweighs the instructions they save.)  Two stages per warp keep
// shared memory small enough for 12 warps per SM; the warp's chain of dependent MMA,
// shuffle and exp2 steps, not the memory latency, sets the pace.
//
// Online softmax in the log2 domain.  The running max of a head only moves when a chunk
// exceeds it by more than 8 (so every weight stays below 2^8 and fp32 sums stay exact
// enough); the accumulator rescale is skipped in the common case where no head moved.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct SAParams {
  const uint16_t* Q;  // [rows, Hq, D]
  const uint16_t* K;  // [total_k, Hkv, D]
  const uint16_t* V;
  const int* indices;  // [rows, k]
  const int* cu_q;     // null for decode (row b is sequence b)
  const int* cu_k;
  int batch;
  long long rows;
  int Hq, Hkv, G, k;
  int nsplit;  // key splits per (row, group); 1 = write final O/LSE
  float scale_log2;
  uint16_t* O;  // [rows, Hq, D] (nsplit == 1)
  float* lse;   // [rows, Hq] or null
  float* part_o;  // [rows, nsplit, Hq, D] (nsplit > 1)
  float* part_ml; // [rows, nsplit, Hq, 4]: max (log2 domain), exact sum, sum of bf16-rounded weights
  const uint8_t* skip_rows;  // optional [rows]: rows another kernel computes (left untouched)
};

// 4-warp CTAs with 2 stages per warp: 3 CTAs, 12 warps per SM.  (Decode launches only a
// thousand warps; 1-warp CTAs with 4 stages each, all resident at once, measured slower.)
constexpr int SA_WARPS = 7;   // warps per CTA (two CTAs per SM: 14 warps, 224 KB of K/V rings at d = 128)
constexpr int SA_STAGES = 2;  // chunks in flight per warp, the one in use included
constexpr int SA_CHUNK = 16;

template <int D, int STAGES>
constexpr int sa_smem_bytes(int warps) {
  return warps * STAGES * 2 * SA_CHUNK * D * 2;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                                  uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
// byte offset of 16-byte segment `seg` of row `row` in a [rows][D] bf16 tile, XOR-swizzled
// so that 8 consecutive rows at one logical segment fall in distinct bank groups
template <int D>
__device__ __forceinline__ uint32_t tile_off(int row, int seg) {
  return (uint32_t)(row * (D * 2) + ((seg ^ (row & 7)) << 4));
}

template <int D, int SA_STAGES, int SA_WARPS>
__global__ void __launch_bounds__(SA_WARPS * 32, 2) sparse_attn_kernel(const SAParams p) {
  constexpr int SEGS = D / 8;                   // 16-byte segments per row
  constexpr int TILE_BYTES = SA_CHUNK * D * 2;  // one K or V chunk
  constexpr int STAGE_BYTES = 2 * TILE_BYTES;
  constexpr int MT = D / 16;                    // m-tiles of O^T, k-steps of S^T
  static_assert(MT % 2 == 0, "two interleaved S chains");
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t my_s = smem_u32(smem + warp * SA_STAGES * STAGE_BYTES);

  // Tasks run KV head by KV head (the head is the slowest index): the warps resident at
  // one time then gather from one head's K/V rows only, a quarter of the K/V bytes, which
  // stays in L2 at 128K context (64 MiB per head) where all four heads' rows would not.
  const long long task = (long long)blockIdx.x * SA_WARPS + warp;
  const long long per_head = p.rows * p.nsplit;
  const int g = (int)(task / per_head);
  if (g >= p.Hkv) return;  // warp-uniform; the kernel has no CTA-wide barrier
  const long long rem = task - (long long)g * per_head;
  const long long row = rem / p.nsplit;
  const int split = (int)(rem % p.nsplit);
  if (p.skip_rows && p.skip_rows[row]) return;  // warp-uniform
  int kbase = 0, vis = 0;
  if (p.cu_q) {
    int lo = 0, hi = p.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if ((long long)p.cu_q[mid] <= row) lo = mid; else hi = mid;
    }
    kbase = p.cu_k[lo];
    vis = causal_vis((int)(row - p.cu_q[lo]), p.cu_q[lo + 1] - p.cu_q[lo], p.cu_k[lo + 1] - kbase);
  } else {
    kbase = p.cu_k[row];
    vis = p.cu_k[row + 1] - kbase;
  }
  const int keys_per_split = p.k / p.nsplit;
  const int* idx = p.indices + row * p.k + split * keys_per_split;
  const int nchunks = keys_per_split / SA_CHUNK;
  const uint16_t* Kg = p.K + (size_t)g * D;
  const uint16_t* Vg = p.V + (size_t)g * D;
  const size_t kv_row_stride = (size_t)p.Hkv * D;

  // Q_g^T as the B operand: b[kk][0..1] for k-step kk (head n = lane/4, d pair (lane%4)*2)
  uint32_t qb[MT][2];
  {
    const int head = lane / 4;
    const bool hv = head < p.G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.Q + ((size_t)row * p.Hq + g * p.G + (hv ? head : 0)) * D);
#pragma unroll
    for (int kk = 0; kk < MT; ++kk) {
      qb[kk][0] = hv ? __ldg(qrow + kk * 8 + (lane % 4)) : 0u;
      qb[kk][1] = hv ? __ldg(qrow + kk * 8 + 4 + (lane % 4)) : 0u;
    }
  }

  // Issues the gather of one chunk into stage st; lane j < 16 holds the index of slot j
  // (lanes 16-31 the same).  Returns the chunk's valid-slot mask, the same in every lane.
  // Eight lanes per row: each copy instruction moves 128-byte pieces (whole lines) of four
  // rows, and a row's slot, validity and address are worked out once for all its pieces.
  auto issue = [&](int st, int my_idx) -> uint32_t {
    const uint32_t kdst = my_s + st * STAGE_BYTES;
    const uint32_t vdst = kdst + TILE_BYTES;
    const int sub = lane >> 3, c = lane & 7;
#pragma unroll
    for (int j = 0; j < SA_CHUNK / 4; ++j) {
      const int r = 4 * j + sub;
      const int s = __shfl_sync(0xffffffffu, my_idx, r);
      const bool valid = (unsigned)s < (unsigned)vis;  // -1 and positions the row cannot see
      const size_t off = valid ? (size_t)(kbase + s) * kv_row_stride + c * 8 : 0;
      const uint32_t o = tile_off<D>(r, c);
#pragma unroll
      for (int h = 0; h < SEGS / 8; ++h) {  // segment c + 8h lands 128 h bytes after segment c
        cp_async_16(kdst + o + h * 128, Kg + off + h * 64, valid);
        cp_async_16(vdst + o + h * 128, Vg + off + h * 64, valid);
      }
    }
    cp_async_commit();
    return __ballot_sync(0xffffffffu, (unsigned)my_idx < (unsigned)vis) & 0xFFFFu;
  };

  float acc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY;  // running max (log2 domain) of heads h0, h1
  float l0 = 0.f, l1 = 0.f;              // this lane's share of the running sums (for the LSE)
  float r0 = 0.f, r1 = 0.f;              // same, of the bf16-rounded weights that multiply V

  // valid-slot masks of the chunks in flight (vmr[0] = the chunk in use next) and the
  // prefetched slot index of the next chunk to issue
  const int slot = lane & 15;
  uint32_t vmr[SA_STAGES - 1];
  int nxt = nchunks > 0 ? __ldg(idx + slot) : -1;
#pragma unroll
  for (int c = 0; c < SA_STAGES - 1; ++c) {
    const int cur = nxt;
    nxt = c + 1 < nchunks ? __ldg(idx + (c + 1) * SA_CHUNK + slot) : -1;
    vmr[c] = c < nchunks ? issue(c, cur) : (cp_async_commit(), 0u);
  }

#pragma unroll 1
  for (int c = 0; c < nchunks; ++c) {
    const int st = c % SA_STAGES;
    uint32_t vnew = 0;
    {
      const int cn = c + SA_STAGES - 1;
      if (cn < nchunks) {
        const int cur = nxt;
        nxt = cn + 1 < nchunks ? __ldg(idx + (cn + 1) * SA_CHUNK + slot) : -1;
        vnew = issue(cn % SA_STAGES, cur);
      } else {
        cp_async_commit();
      }
    }
    cp_async_wait<SA_STAGES - 1>();
    __syncwarp();
    const uint32_t kt = my_s + st * STAGE_BYTES;
    const uint32_t vt = kt + TILE_BYTES;

    // ---- S^T = K_chunk . Q^T, two interleaved accumulator chains
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < MT; kk += 2) {
      uint32_t a0, a1, a2, a3, e0, e1, e2, e3;
      ldmatrix_x4(kt + tile_off<D>(lane & 15, kk * 2 + (lane >> 4)), a0, a1, a2, a3);
      ldmatrix_x4(kt + tile_off<D>(lane & 15, (kk + 1) * 2 + (lane >> 4)), e0, e1, e2, e3);
      mma_bf16_16816(sa, a0, a1, a2, a3, qb[kk][0], qb[kk][1]);
      mma_bf16_16816(sb, e0, e1, e2, e3, qb[kk + 1][0], qb[kk + 1][1]);
    }
    // keys of this lane: q0 = lane/4, q1 = lane/4 + 8; heads h0 = 2*(lane%4), h1 = h0 + 1
    const uint32_t vm = vmr[0];
    const bool v0 = (vm >> (lane >> 2)) & 1u;
    const bool v1 = (vm >> ((lane >> 2) + 8)) & 1u;
    const float x00 = v0 ? (sa[0] + sb[0]) * p.scale_log2 : -INFINITY;  // (q0, h0)
    const float x01 = v0 ? (sa[1] + sb[1]) * p.scale_log2 : -INFINITY;  // (q0, h1)
    const float x10 = v1 ? (sa[2] + sb[2]) * p.scale_log2 : -INFINITY;  // (q1, h0)
    const float x11 = v1 ? (sa[3] + sb[3]) * p.scale_log2 : -INFINITY;  // (q1, h1)
    float cm0 = fmaxf(x00, x10), cm1 = fmaxf(x01, x11);
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      cm0 = fmaxf(cm0, __shfl_xor_sync(0xffffffffu, cm0, o));
      cm1 = fmaxf(cm1, __shfl_xor_sync(0xffffffffu, cm1, o));
    }
    const bool up0 = cm0 > m0 + 8.f, up1 = cm1 > m1 + 8.f;
    if (__any_sync(0xffffffffu, up0 || up1)) {
      const float al0 = up0 ? exp2f(m0 - cm0) : 1.f, al1 = up1 ? exp2f(m1 - cm1) : 1.f;
      if (up0) m0 = cm0;
      if (up1) m1 = cm1;
      l0 *= al0;
      l1 *= al1;
      r0 *= al0;
      r1 *= al1;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        acc[mt][0] *= al0;
        acc[mt][1] *= al1;
        acc[mt][2] *= al0;
        acc[mt][3] *= al1;
      }
    }
    const float mu0 = m0 == -INFINITY ? 0.f : m0, mu1 = m1 == -INFINITY ? 0.f : m1;
    const float p00 = exp2f(x00 - mu0), p01 = exp2f(x01 - mu1);
    const float p10 = exp2f(x10 - mu0), p11 = exp2f(x11 - mu1);
    l0 += p00 + p10;
    l1 += p01 + p11;
    // O is normalised by the sum of the weights exactly as they enter the PV product
    const uint32_t pk0 = pack_bf16x2(p00, p01), pk1 = pack_bf16x2(p10, p11);
    r0 += __uint_as_float(pk0 << 16) + __uint_as_float(pk1 << 16);
    r1 += __uint_as_float(pk0 & 0xFFFF0000u) + __uint_as_float(pk1 & 0xFFFF0000u);
    // ---- O^T += V^T . P^T
    const uint32_t pb0 = movmatrix_trans(pk0);  // keys 0-7
    const uint32_t pb1 = movmatrix_trans(pk1);  // keys 8-15
    const int vrow = (lane & 7) + ((lane >> 4) << 3);
    const int vseg_off = (lane >> 3) & 1;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a0, a1, a2, a3;
      ldmatrix_x4_trans(vt + tile_off<D>(vrow, mt * 2 + vseg_off), a0, a1, a2, a3);
      mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
    }
#pragma unroll
    for (int j = 0; j + 1 < SA_STAGES - 1; ++j) vmr[j] = vmr[j + 1];
    vmr[SA_STAGES - 2] = vnew;
    __syncwarp();  // stage st is refilled by the next iteration's issue
  }
  cp_async_wait<0>();

  // ---- finish: reduce the sums over the lanes holding the same heads
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    r0 += __shfl_xor_sync(0xffffffffu, r0, o);
    r1 += __shfl_xor_sync(0xffffffffu, r1, o);
  }
  const int h0 = 2 * (lane % 4), h1 = h0 + 1;
  if (p.nsplit == 1) {
    const float inv0 = r0 > 0.f ? 1.f / r0 : 0.f, inv1 = r1 > 0.f ? 1.f / r1 : 0.f;
    uint16_t* orow = p.O + ((size_t)row * p.Hq + g * p.G) * D;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int d0 = mt * 16 + lane / 4;
      if (h0 < p.G) {
        orow[h0 * D + d0] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][0] * inv0));
        orow[h0 * D + d0 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][2] * inv0));
      }
      if (h1 < p.G) {
        orow[h1 * D + d0] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][1] * inv1));
        orow[h1 * D + d0 + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[mt][3] * inv1));
      }
    }
    if (p.lse && lane < 4) {
      const float ln2 = 0.69314718055994531f;
      if (h0 < p.G) p.lse[row * p.Hq + g * p.G + h0] = l0 > 0.f ? (m0 + log2f(l0)) * ln2 : -INFINITY;
      if (h1 < p.G) p.lse[row * p.Hq + g * p.G + h1] = l1 > 0.f ? (m1 + log2f(l1)) * ln2 : -INFINITY;
    }
  } else {
    float* po = p.part_o + (((size_t)row * p.nsplit + split) * p.Hq + g * p.G) * D;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      const int d0 = mt * 16 + lane / 4;
      if (h0 < p.G) {
        po[h0 * D + d0] = acc[mt][0];
        po[h0 * D + d0 + 8] = acc[mt][2];
      }
      if (h1 < p.G) {
        po[h1 * D + d0] = acc[mt][1];
        po[h1 * D + d0 + 8] = acc[mt][3];
      }
    }
    if (lane < 4) {
      float* pml = p.part_ml + (((size_t)row * p.nsplit + split) * p.Hq + g * p.G) * 4;
      if (h0 < p.G) *reinterpret_cast<float4*>(pml + h0 * 4) = make_float4(m0, l0, r0, 0.f);
      if (h1 < p.G) *reinterpret_cast<float4*>(pml + h1 * 4) = make_float4(m1, l1, r1, 0.f);
    }
  }
}

// Merges the per-split partial softmax states of decode: one warp per (row, head, 32 of the
// D output dims), lane s holding split s's (max, sum, weight sum) (nsplit <= 32).  Every
// load of the warp (its splits' 32 dims of O, and the states) is issued before any of the
// merge arithmetic, so the kernel costs about one memory round trip.
template <int D>
__global__ void decode_combine_kernel(const float* part_o, const float* part_ml, int rows, int Hq, int nsplit,
                                      uint16_t* O, float* lse) {
  pdl_wait();
  pdl_trigger();
  constexpr int PARTS = D / 32;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (gw >= rows * Hq * PARTS) return;
  const int part = gw % PARTS, rh = gw / PARTS;
  const int row = rh / Hq, h = rh % Hq;
  float v[32];
#pragma unroll
  for (int s = 0; s < 32; ++s)
    v[s] = s < nsplit ? part_o[(((size_t)row * nsplit + s) * Hq + h) * D + part * 32 + lane] : 0.f;
  float m = -INFINITY, l = 0.f, rr = 0.f;
  if (lane < nsplit) {
    const float4 ml = *reinterpret_cast<const float4*>(part_ml + (((size_t)row * nsplit + lane) * Hq + h) * 4);
    m = ml.x;
    l = ml.y;
    rr = ml.z;
  }
  float M = m;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  const float Mu = M == -INFINITY ? 0.f : M;
  const float f = (m == -INFINITY) ? 0.f : exp2f(m - Mu);
  float L = l * f, R = rr * f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    L += __shfl_xor_sync(0xffffffffu, L, o);
    R += __shfl_xor_sync(0xffffffffu, R, o);
  }
  float acc = 0.f;
#pragma unroll
  for (int s = 0; s < 32; ++s) acc += __shfl_sync(0xffffffffu, f, s) * v[s];
  const float inv = R > 0.f ? 1.f / R : 0.f;
  O[((size_t)row * Hq + h) * D + part * 32 + lane] = __bfloat16_as_ushort(__float2bfloat16_rn(acc * inv));
  if (lse && part == 0 && lane == 0) lse[(size_t)row * Hq + h] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace dsa

namespace dsa_host {

template <int D, int STAGES, int WARPS>
static int sa_launch_d(const dsa::SAParams& p, long long tasks, cudaStream_t stream) {
  const long long blocks = (tasks + WARPS - 1) / WARPS;
  const int smem = dsa::sa_smem_bytes<D, STAGES>(WARPS);
  static DeviceFlag done;
  if (!done) {
    cudaError_t e_ = cudaFuncSetAttribute(dsa::sparse_attn_kernel<D, STAGES, WARPS>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    // several CTAs per SM need the largest shared-memory carveout
    if (e_ == cudaSuccess)
      e_ = cudaFuncSetAttribute(dsa::sparse_attn_kernel<D, STAGES, WARPS>,
                                cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e_ != cudaSuccess) return cuda_fail(e_);
    done = true;
  }
  return launch_pdl(false, dsa::sparse_attn_kernel<D, STAGES, WARPS>, dim3((unsigned)blocks), dim3(WARPS * 32),
                    (size_t)smem, stream, p);
}

static int sa_launch_common(dsa::SAParams& p, int d, cudaStream_t stream) {
  const long long tasks = p.rows * p.Hkv * p.nsplit;
  if (tasks <= 0) return DSA_OK;
  return d == 128 ? sa_launch_d<128, dsa::SA_STAGES, dsa::SA_WARPS>(p, tasks, stream)
                  : sa_launch_d<64, dsa::SA_STAGES, dsa::SA_WARPS>(p, tasks, stream);
}

int sparse_attn_prefill_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                               const int* cu_k, int batch, long long total_q, int Hq, int Hkv, int d, int k,
                               float scale, void* O, float* lse, cudaStream_t stream, const uint8_t* skip_rows) {
  dsa::SAParams p{};
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.indices = indices;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.rows = total_q;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.k = k;
  p.nsplit = 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse;
  p.skip_rows = skip_rows;
  return sa_launch_common(p, d, stream);
}

int decode_nsplit(int k) {
  int ns = k / 128;  // 128 keys per split; <= 32 for k <= 4096 (the combine kernel's lane-per-split)
  if (ns < 1) ns = 1;
  while (ns > 1 && (k % (ns * dsa::SA_CHUNK)) != 0) --ns;
  return ns;
}

size_t decode_workspace_bytes(int batch, int Hq, int d, int k) {
  const int ns = decode_nsplit(k);
  return (size_t)batch * ns * Hq * ((size_t)d + 4) * sizeof(float) + 256;
}

int sparse_attn_decode_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_k,
                              int batch, int Hq, int Hkv, int d, int k, float scale, void* O, float* lse,
                              void* ws, cudaStream_t stream) {
  dsa::SAParams p{};
  p.Q = static_cast<const uint16_t*>(Q);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.indices = indices;
  p.cu_q = nullptr;
  p.cu_k = cu_k;
  p.batch = batch;
  p.rows = batch;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.k = k;
  p.nsplit = decode_nsplit(k);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse;
  if (p.nsplit == 1) return sa_launch_common(p, d, stream);
  p.part_o = static_cast<float*>(ws);
  p.part_ml = p.part_o + (size_t)batch * p.nsplit * Hq * d;
  int st = sa_launch_common(p, d, stream);
  if (st != DSA_OK) return st;
  const int warps = batch * Hq * (d / 32);
  const int threads = 256;
  const int blocks = (warps * 32 + threads - 1) / threads;
  const float* part_o = p.part_o;
  const float* part_ml = p.part_ml;
  uint16_t* O_ = p.O;
  const int nsplit = p.nsplit;
  if (d == 128)
    return launch_pdl(true, dsa::decode_combine_kernel<128>, dim3(blocks), dim3(threads), 0, stream, part_o, part_ml, batch,
                      Hq, nsplit, O_, lse);
  return launch_pdl(true, dsa::decode_combine_kernel<64>, dim3(blocks), dim3(threads), 0, stream, part_o, part_ml, batch,
                    Hq, nsplit, O_, lse);
}

}  // namespace dsa_host
