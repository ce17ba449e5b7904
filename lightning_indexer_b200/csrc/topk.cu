// Deterministic per-row top-k over indexer scores (sm_100a, CUDA cores).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1 (each token keeps
// its 2048 most relevant positions) and section 8 (top-k must be deterministic so that
// training and inference select identical sets).
//
// Selection rule: the k largest scores among the visible positions; equal scores are
// ranked by the lower position (+0.0 == -0.0).  Output: ascending positions, -1 padded.
//
// Method (one thread block per row, no global atomics, no data-dependent ordering):
//   1. three radix-histogram passes (11 + 11 + 10 bits of the order-preserving uint32
//      key) find the exact k-th largest key K* and how many of the ties at K* to take;
//   2. one ordered compaction pass: position s is selected if key(s) > K*, or
//      key(s) == K* and fewer than `remaining` ties precede it.  Its output slot is
//      (#keys > K* before s) + min(#ties before s, remaining), so the output is the
//      ascending position list and is bit-for-bit reproducible.
#include "common.cuh"

namespace dsa {

struct TopkParams {
  const float* scores;
  long long ld;
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin;
  int k;
  int* indices;
};

template <int BLOCK>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    constexpr int NW = BLOCK / 32;
    uint32_t s = lane < NW ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < NW) warp_sums[lane] = s;  // inclusive prefix of warp totals
    if (lane == NW - 1) *total = s;
  }
  __syncthreads();
  const uint32_t before = (warp > 0 ? warp_sums[warp - 1] : 0u) + x - v;
  __syncthreads();  // warp_sums may be reused by the caller right away
  return before;
}

// Finds the bin holding the `remaining`-th largest element of the histogram: the bin b
// with (#elements in bins > b) < remaining <= (#elements in bins >= b).
template <int BLOCK, int NBINS>
__device__ __forceinline__ void find_bin(const uint32_t* hist, uint32_t remaining, uint32_t* warp_sums,
                                         uint32_t* scratch, uint32_t* out_bin, uint32_t* out_above) {
  constexpr int PER = NBINS / BLOCK;  // bins per thread, visited from the top
  static_assert(PER >= 1 && NBINS % BLOCK == 0, "bins per thread");
  uint32_t c[PER];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = hist[NBINS - 1 - (threadIdx.x * PER + j)];
    local += c[j];
  }
  uint32_t above = block_excl_scan<BLOCK>(local, warp_sums, scratch);
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    if (above < remaining && above + c[j] >= remaining) {
      *out_bin = NBINS - 1 - (threadIdx.x * PER + j);
      *out_above = above;
    }
    above += c[j];
  }
  __syncthreads();
}

template <int BLOCK>
__global__ void __launch_bounds__(BLOCK) topk_kernel(const TopkParams p) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t s_total, s_bin, s_above;

  const long long row = p.row_begin + blockIdx.x;
  // sequence of this row (cu_q is small; binary search)
  int lo = 0, hi = p.batch;  // find b with cu_q[b] <= row < cu_q[b+1]
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)p.cu_q[mid] <= row) lo = mid; else hi = mid;
  }
  const int b = lo;
  const int i = (int)(row - p.cu_q[b]);
  const int Lq = p.cu_q[b + 1] - p.cu_q[b];
  const int Lk = p.cu_k[b + 1] - p.cu_k[b];
  const int vis = min(max(i + Lk - Lq + 1, 0), Lk);
  const int k = p.k;
  int* out = p.indices + (long long)blockIdx.x * k;
  const float* src = p.scores + (long long)blockIdx.x * p.ld;

  if (vis <= k) {
    for (int j = threadIdx.x; j < k; j += BLOCK) out[j] = j < vis ? j : -1;
    return;
  }

  const int nvec = vis / 4;  // float4 groups; the ragged tail is handled one by one
  const float4* src4 = reinterpret_cast<const float4*>(src);

  uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
  // ---------------------------------------------------------------- radix passes
#pragma unroll 1
  for (int level = 0; level < 3; ++level) {
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const uint32_t bmask = level == 2 ? 1023u : 2047u;
    for (int j = threadIdx.x; j < 2048; j += BLOCK) hist[j] = 0;
    __syncthreads();
#pragma unroll 4
    for (int v = threadIdx.x; v < nvec; v += BLOCK) {
      const float4 x = __ldg(src4 + v);
      const uint32_t k0 = float_order_key(x.x), k1 = float_order_key(x.y);
      const uint32_t k2 = float_order_key(x.z), k3 = float_order_key(x.w);
      if ((k0 & pmask) == prefix) atomicAdd(&hist[(k0 >> shift) & bmask], 1u);
      if ((k1 & pmask) == prefix) atomicAdd(&hist[(k1 >> shift) & bmask], 1u);
      if ((k2 & pmask) == prefix) atomicAdd(&hist[(k2 >> shift) & bmask], 1u);
      if ((k3 & pmask) == prefix) atomicAdd(&hist[(k3 >> shift) & bmask], 1u);
    }
    for (int s = nvec * 4 + threadIdx.x; s < vis; s += BLOCK) {
      const uint32_t kk = float_order_key(__ldg(src + s));
      if ((kk & pmask) == prefix) atomicAdd(&hist[(kk >> shift) & bmask], 1u);
    }
    __syncthreads();
    if (level < 2)
      find_bin<BLOCK, 2048>(hist, remaining, warp_sums, &s_total, &s_bin, &s_above);
    else
      find_bin<BLOCK, 1024>(hist, remaining, warp_sums, &s_total, &s_bin, &s_above);
    prefix |= s_bin << shift;
    pmask |= bmask << shift;
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t kstar = prefix;  // exact key of the k-th largest score
  const uint32_t n_gt_total = (uint32_t)k - remaining;

  // ---------------------------------------------------------------- ordered compaction
  constexpr int ITEMS = 4;
  uint32_t base_gt = 0, base_tie = 0;
#pragma unroll 1
  for (int start = 0; start < vis; start += BLOCK * ITEMS) {
    const int s0 = start + threadIdx.x * ITEMS;
    uint32_t key[ITEMS];
    if (s0 + ITEMS <= vis) {
      const float4 x = __ldg(src4 + s0 / 4);
      key[0] = float_order_key(x.x);
      key[1] = float_order_key(x.y);
      key[2] = float_order_key(x.z);
      key[3] = float_order_key(x.w);
    } else {
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) key[j] = (s0 + j < vis) ? float_order_key(__ldg(src + s0 + j)) : 0u;
    }
    uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
      const bool valid = s0 + j < vis;
      n_gt += (valid && key[j] > kstar);
      n_eq += (valid && key[j] == kstar);
    }
    const uint32_t packed = (n_gt << 16) | n_eq;  // each field <= BLOCK*ITEMS < 65536
    const uint32_t excl = block_excl_scan<BLOCK>(packed, warp_sums, &s_total);
    uint32_t gt_before = base_gt + (excl >> 16);
    uint32_t eq_before = base_tie + (excl & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < ITEMS; ++j) {
      if (s0 + j >= vis) break;
      if (key[j] > kstar) {
        out[gt_before + min(eq_before, remaining)] = s0 + j;
        ++gt_before;
      } else if (key[j] == kstar) {
        if (eq_before < remaining) out[gt_before + eq_before] = s0 + j;
        ++eq_before;
      }
    }
    const uint32_t tot = s_total;
    base_gt += tot >> 16;
    base_tie += tot & 0xFFFFu;
    __syncthreads();  // s_total is rewritten by the next scan
    if (base_gt == n_gt_total && base_tie >= remaining) break;  // every selected position found
  }
}

}  // namespace dsa

namespace dsa_host {

int topk_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                long long row_begin, long long row_end, int k, int* indices, cudaStream_t stream) {
  const long long rows = row_end - row_begin;
  if (rows <= 0) return DSA_OK;
  dsa::TopkParams p;
  p.scores = scores;
  p.ld = ld;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.row_begin = row_begin;
  p.k = k;
  p.indices = indices;
  if (rows > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  dsa::topk_kernel<1024><<<(unsigned)rows, 1024, 0, stream>>>(p);
  return last_launch_status();
}

}  // namespace dsa_host
