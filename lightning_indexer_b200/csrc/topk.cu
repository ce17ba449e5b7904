// Deterministic per-row top-k over indexer scores (sm_100a, CUDA cores).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1 (each token keeps
// its 2048 most relevant positions) and section 8 (top-k must be deterministic so that
// training and inference select identical sets).
//
// Selection rule: the k largest scores among the visible positions; equal scores are
// ranked by the lower position (+0.0 == -0.0).  Output: ascending positions, -1 padded.
//
// Method.  A row is split over a cluster of C thread blocks (C = 1, 2, 4 or 8), each
// owning a contiguous segment.  Scores map to order-preserving uint32 keys.
//   1. A lower bound T on the k-th largest key is estimated from a fixed strided sample
//      of the row (the same 1024 positions in every block, so no communication), with a
//      safety margin.  One global pass compacts the keys >= T of each segment, in
//      position order, into a shared-memory candidate list.  The cluster checks that at
//      least k keys passed and that every block's list fit; the estimate only decides
//      how much is read, never what is selected.
//   2. Otherwise (an unlucky sample, or a row with huge ties): an exact histogram of the
//      top 11 key bits (summed over the cluster through distributed shared memory) gives
//      the threshold bin b1; the keys with bin >= b1 become the candidates if they fit,
//      else every later step re-reads the segment from global memory.
//   3. Radix levels (11 + 11 + 10 bits) over the candidates give the exact k-th key K*
//      and how many ties at K* to take (`remaining`).
//   4. Ordered output: position s is selected if key > K*, or key == K* and fewer than
//      `remaining` ties precede it in the row.  Each block learns from the lower-ranked
//      blocks how many keys > K* and ties come before its segment, so its slots are
//      (#keys > K* before s) + min(#ties before s, remaining): ascending and
//      bit-reproducible.  No global atomics are used anywhere.
#include <algorithm>
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

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
  int only_marked;  // exact kernel: process only the rows the fast kernel marked with -2
  int* flag_reset = nullptr;  // marked-row kernel: cleared (set to 0) by the launch
};

constexpr int TOPK_THREADS = 1024;
constexpr int TOPK_CAP = 11264;  // candidates kept in shared memory per block

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

// The bin b with (#elements in bins > b) < remaining <= (#elements in bins >= b).
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

template <int C>
__device__ __forceinline__ void cluster_sync_all() {
  if constexpr (C > 1) cg::this_cluster().sync();
  else __syncthreads();
}

struct TopkSmem {
  uint32_t cand_key[TOPK_CAP];
  int cand_pos[TOPK_CAP];
  uint32_t hist[2][2048];  // per level parity (remote blocks read them)
  uint32_t ghist[2048];    // cluster-wide sum
  uint32_t warp_sums[32];
  uint32_t total, bin, above;
  uint32_t flag;     // this block's candidates overflow TOPK_CAP
  uint32_t counts[2];  // (#keys > K*, #ties) of this block's segment
  uint32_t dmax;
};

// The exact selection of one row (by a cluster of C blocks).
template <int C>
__device__ void exact_row_select(const TopkParams& p, TopkSmem& S, const long long row) {
  constexpr int B = TOPK_THREADS;
  const int rank = (C > 1) ? (int)cg::this_cluster().block_rank() : 0;
  int lo = 0, hi = p.batch;
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
  int* out = p.indices + (row - p.row_begin) * k;
  const float* src = p.scores + (row - p.row_begin) * p.ld;

  // (uniform over the cluster: every block reads out[0] before any block writes the row)
  if (p.only_marked && __ldg(out) != -2) return;
  if (vis <= k) {  // uniform over the cluster: no cluster barrier is reached by anyone
    if (rank == 0)
      for (int j = threadIdx.x; j < k; j += B) out[j] = j < vis ? j : -1;
    return;
  }
  // this block's segment [s_lo, s_hi), 4-aligned starts
  const int seg = ((vis + C - 1) / C + 3) & ~3;
  const int s_lo = min(rank * seg, vis), s_hi = min(s_lo + seg, vis);

  auto reduce_hist = [&](int par, int nbins) -> const uint32_t* {
    if constexpr (C == 1) {
      return S.hist[par];
    } else {
      auto cl = cg::this_cluster();
      for (int j = threadIdx.x; j < nbins; j += B) {
        uint32_t t = 0;
#pragma unroll
        for (int r = 0; r < C; ++r) t += cl.map_shared_rank(&S.hist[par][0], r)[j];
        S.ghist[j] = t;
      }
      __syncthreads();
      return S.ghist;
    }
  };
  constexpr int ITEMS = 16;  // contiguous elements per thread per tile (4 x float4 in flight)
  // loads ITEMS keys of positions [s0, s0 + ITEMS) clipped to the segment (s0 4-aligned)
  auto load_keys = [&](int s0, uint32_t* key) {
    if (s0 + ITEMS <= s_hi) {
      float4 x[ITEMS / 4];
#pragma unroll
      for (int u = 0; u < ITEMS / 4; ++u) x[u] = __ldg(reinterpret_cast<const float4*>(src + s0) + u);
#pragma unroll
      for (int u = 0; u < ITEMS / 4; ++u) {
        key[4 * u + 0] = float_order_key(x[u].x);
        key[4 * u + 1] = float_order_key(x[u].y);
        key[4 * u + 2] = float_order_key(x[u].z);
        key[4 * u + 3] = float_order_key(x[u].w);
      }
    } else {
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) key[j] = (s0 + j < s_hi) ? float_order_key(__ldg(src + s0 + j)) : 0u;
    }
  };
  // ordered compaction of the segment's keys with pred(key) into the candidate list;
  // returns the count (which may exceed TOPK_CAP: nothing is written past the end)
  auto compact = [&](auto&& pred) -> uint32_t {
    uint32_t base = 0;
    for (int start = s_lo; start < s_hi; start += B * ITEMS) {
      const int s0 = start + threadIdx.x * ITEMS;
      uint32_t key[ITEMS];
      load_keys(s0, key);
      uint32_t n = 0;
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) n += (s0 + j < s_hi && pred(key[j]));
      uint32_t pos = base + block_excl_scan<B>(n, S.warp_sums, &S.total);
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        if (s0 + j < s_hi && pred(key[j])) {
          if (pos < (uint32_t)TOPK_CAP) {
            S.cand_key[pos] = key[j];
            S.cand_pos[pos] = s0 + j;
          }
          ++pos;
        }
      }
      base += S.total;
      __syncthreads();  // S.total is rewritten by the next scan
    }
    return base;
  };
  // cluster-wide: (sum of counts >= k) and (every count <= TOPK_CAP)
  auto cluster_ok = [&](uint32_t cnt) -> bool {
    if (threadIdx.x == 0) S.counts[0] = cnt;
    cluster_sync_all<C>();
    uint32_t tot = 0;
    bool fit = true;
    if constexpr (C == 1) {
      tot = S.counts[0];
      fit = tot <= (uint32_t)TOPK_CAP;
    } else {
      auto cl = cg::this_cluster();
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t c = *cl.map_shared_rank(&S.counts[0], r);
        tot += c;
        fit = fit && c <= (uint32_t)TOPK_CAP;
      }
    }
    cluster_sync_all<C>();  // counts[0] is rewritten later
    return fit && tot >= (uint32_t)k;
  };

  uint32_t remaining = (uint32_t)k;
  uint32_t prefix = 0, pmask = 0;
  int first_level = 0;
  bool in_smem = false;
  int ncand = 0;
  const uint32_t* gh = nullptr;

  // ---------------------------------------------------------------- 1. sampled threshold
  {
    constexpr int NS = 1024;  // == B: one sample per thread
    uint32_t T = 0;
    if (vis > C * (TOPK_CAP / 2)) {
      // expected sampled keys above the k-th largest, and a margin of ~4 sigma + 8
      const float m = (float)k * (float)NS / (float)vis;
      const int r_low = min(NS, (int)ceilf(1.5f * m + 4.f * sqrtf(m) + 8.f));
      const long long pos = ((2LL * threadIdx.x + 1) * vis) / (2LL * NS);
      const uint32_t sk = float_order_key(__ldg(src + pos));
      // the r_low-th largest sampled key, to 22 bits, by two radix levels over the sample
      uint32_t sp = 0, sm = 0, rem = (uint32_t)r_low;
#pragma unroll 1
      for (int lv = 0; lv < 2; ++lv) {
        const int shift = lv == 0 ? 21 : 10;
        for (int j = threadIdx.x; j < 2048; j += B) S.ghist[j] = 0;
        __syncthreads();
        if ((sk & sm) == sp) atomicAdd(&S.ghist[(sk >> shift) & 2047u], 1u);
        __syncthreads();
        find_bin<B, 2048>(S.ghist, rem, S.warp_sums, &S.total, &S.bin, &S.above);
        sp |= S.bin << shift;
        sm |= 2047u << shift;
        rem -= S.above;
      }
      T = sp;  // every sampled key in the top r_low is >= T
    }
    const uint32_t cnt = compact([&](uint32_t kk) { return kk >= T; });
    in_smem = cluster_ok(cnt);
    ncand = in_smem ? (int)cnt : 0;
  }

  if (!in_smem) {
    // ---------------------------------------------------------------- 2. exact level 1
    for (int j = threadIdx.x; j < 2048; j += B) S.hist[0][j] = 0;
    __syncthreads();
    {
      const int v_lo = s_lo / 4, v_hi = s_hi / 4;  // whole float4 groups inside the segment
      const float4* src4 = reinterpret_cast<const float4*>(src);
      int v = v_lo + threadIdx.x;
      for (; v + 3 * B < v_hi; v += 4 * B) {
        float4 x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = __ldg(src4 + v + u * B);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          atomicAdd(&S.hist[0][float_order_key(x[u].x) >> 21], 1u);
          atomicAdd(&S.hist[0][float_order_key(x[u].y) >> 21], 1u);
          atomicAdd(&S.hist[0][float_order_key(x[u].z) >> 21], 1u);
          atomicAdd(&S.hist[0][float_order_key(x[u].w) >> 21], 1u);
        }
      }
      for (; v < v_hi; v += B) {
        const float4 x = __ldg(src4 + v);
        atomicAdd(&S.hist[0][float_order_key(x.x) >> 21], 1u);
        atomicAdd(&S.hist[0][float_order_key(x.y) >> 21], 1u);
        atomicAdd(&S.hist[0][float_order_key(x.z) >> 21], 1u);
        atomicAdd(&S.hist[0][float_order_key(x.w) >> 21], 1u);
      }
      for (int s = v_hi * 4 + threadIdx.x; s < s_hi; s += B)
        atomicAdd(&S.hist[0][float_order_key(__ldg(src + s)) >> 21], 1u);
    }
    cluster_sync_all<C>();
    gh = reduce_hist(0, 2048);
    find_bin<B, 2048>(gh, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    const uint32_t b1 = S.bin;
    remaining -= S.above;
    prefix = b1 << 21;
    pmask = 0xFFE00000u;
    first_level = 1;
    const uint32_t cnt = compact([&](uint32_t kk) { return (kk >> 21) >= b1; });
    // here the count is >= remaining by construction; only the fit matters
    if (threadIdx.x == 0) S.counts[0] = cnt;
    cluster_sync_all<C>();
    in_smem = true;
    if constexpr (C == 1) {
      in_smem = S.counts[0] <= (uint32_t)TOPK_CAP;
    } else {
      auto cl = cg::this_cluster();
#pragma unroll
      for (int r = 0; r < C; ++r) in_smem = in_smem && (*cl.map_shared_rank(&S.counts[0], r) <= (uint32_t)TOPK_CAP);
    }
    cluster_sync_all<C>();
    ncand = in_smem ? (int)cnt : 0;
  }

  // visits every element of the block's source in position order: f(key, position)
  auto for_each_key = [&](auto&& f) {
    if (in_smem) {
      for (int j = threadIdx.x; j < ncand; j += B) f(S.cand_key[j], S.cand_pos[j]);
    } else {
      for (int s = s_lo + threadIdx.x; s < s_hi; s += B) f(float_order_key(__ldg(src + s)), s);
    }
  };

  // ---------------------------------------------------------------- levels 2 and 3
#pragma unroll 1
  for (int level = first_level; level < 3; ++level) {
    const int par = level & 1;
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const uint32_t bmask = level == 2 ? 1023u : 2047u;
    for (int j = threadIdx.x; j < 2048; j += B) S.hist[par][j] = 0;
    __syncthreads();
    for_each_key([&](uint32_t kk, int) {
      if ((kk & pmask) == prefix) atomicAdd(&S.hist[par][(kk >> shift) & bmask], 1u);
    });
    cluster_sync_all<C>();
    gh = reduce_hist(par, level == 2 ? 1024 : 2048);
    if (level < 2)
      find_bin<B, 2048>(gh, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    else
      find_bin<B, 1024>(gh, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    prefix |= S.bin << shift;
    pmask |= bmask << shift;
    remaining -= S.above;
  }
  const uint32_t kstar = prefix;

  // ---------------------------------------------------------------- ordered output
  // counts of this block, then the counts of all lower-ranked blocks of the cluster
  uint32_t base_gt = 0, base_tie = 0;
  if constexpr (C > 1) {
    uint32_t ngt = 0, neq = 0;
    for_each_key([&](uint32_t kk, int) {
      ngt += kk > kstar;
      neq += kk == kstar;
    });
    block_excl_scan<B>(ngt, S.warp_sums, &S.total);
    const uint32_t tot_gt = S.total;
    __syncthreads();
    block_excl_scan<B>(neq, S.warp_sums, &S.total);
    if (threadIdx.x == 0) {
      S.counts[0] = tot_gt;
      S.counts[1] = S.total;
    }
    cluster_sync_all<C>();
    auto cl = cg::this_cluster();
    for (int r = 0; r < rank; ++r) {
      const uint32_t* rc = cl.map_shared_rank(&S.counts[0], r);
      base_gt += rc[0];
      base_tie += rc[1];
    }
  }
  if (in_smem) {
    constexpr int IT = 4;
    for (int start = 0; start < ncand; start += B * IT) {
      const int j0 = start + threadIdx.x * IT;
      uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
      for (int j = 0; j < IT; ++j) {
        if (j0 + j < ncand) {
          n_gt += S.cand_key[j0 + j] > kstar;
          n_eq += S.cand_key[j0 + j] == kstar;
        }
      }
      const uint32_t excl = block_excl_scan<B>((n_gt << 16) | n_eq, S.warp_sums, &S.total);
      uint32_t gt_before = base_gt + (excl >> 16), eq_before = base_tie + (excl & 0xFFFFu);
#pragma unroll
      for (int j = 0; j < IT; ++j) {
        if (j0 + j >= ncand) break;
        const uint32_t kk = S.cand_key[j0 + j];
        if (kk > kstar) {
          out[gt_before + min(eq_before, remaining)] = S.cand_pos[j0 + j];
          ++gt_before;
        } else if (kk == kstar) {
          if (eq_before < remaining) out[gt_before + eq_before] = S.cand_pos[j0 + j];
          ++eq_before;
        }
      }
      base_gt += S.total >> 16;
      base_tie += S.total & 0xFFFFu;
      __syncthreads();
    }
  } else {
    for (int start = s_lo; start < s_hi; start += B * ITEMS) {
      const int s0 = start + threadIdx.x * ITEMS;
      uint32_t key[ITEMS];
      load_keys(s0, key);
      uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        n_gt += (s0 + j < s_hi && key[j] > kstar);
        n_eq += (s0 + j < s_hi && key[j] == kstar);
      }
      // per-thread counts <= 16 and block totals <= 16384 fit the packed 16-bit fields
      const uint32_t excl = block_excl_scan<B>((n_gt << 16) | n_eq, S.warp_sums, &S.total);
      uint32_t gt_before = base_gt + (excl >> 16), eq_before = base_tie + (excl & 0xFFFFu);
#pragma unroll
      for (int j = 0; j < ITEMS; ++j) {
        if (s0 + j >= s_hi) break;
        if (key[j] > kstar) {
          out[gt_before + min(eq_before, remaining)] = s0 + j;
          ++gt_before;
        } else if (key[j] == kstar) {
          if (eq_before < remaining) out[gt_before + eq_before] = s0 + j;
          ++eq_before;
        }
      }
      base_gt += S.total >> 16;
      base_tie += S.total & 0xFFFFu;
      __syncthreads();
    }
  }
  // no block may leave while another still reads its shared memory
  if constexpr (C > 1) cg::this_cluster().sync();
}

template <int C>
__global__ void __launch_bounds__(TOPK_THREADS) topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  exact_row_select<C>(p, S, p.row_begin + blockIdx.x / C);
}

// The exact selection of the rows a one-block-per-row kernel marked with -2 (p.only_marked
// set): block b first collects the marked rows of its contiguous share (<= TOPK_THREADS
// rows, one flag read per thread), then selects them one after the other.
__global__ void __launch_bounds__(TOPK_THREADS) topk_marked_kernel(const TopkParams p, long long rows) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  __shared__ int marked[TOPK_THREADS];
  __shared__ int nmarked;
  const long long per = (rows + gridDim.x - 1) / gridDim.x;
  const long long r0 = blockIdx.x * per, r1 = min(rows, r0 + per);
  if (threadIdx.x == 0) nmarked = 0;
  __syncthreads();
  if (r0 + threadIdx.x < r1 && __ldg(p.indices + (r0 + threadIdx.x) * p.k) == -2)
    marked[atomicAdd(&nmarked, 1)] = (int)threadIdx.x;
  __syncthreads();
  const int n = nmarked;
  if (p.flag_reset && blockIdx.x == 0 && threadIdx.x == 0) *p.flag_reset = 0;
  for (int j = 0; j < n; ++j) exact_row_select<1>(p, S, p.row_begin + r0 + marked[j]);
}

// ======================================================================================
// Fast path.  512 threads, two blocks per SM.  A sampled lower bound T is taken first (the
// same 2048 strided positions in every block of the row); one streaming pass then
// appends the keys >= T of the block's segment to a shared-memory candidate list with
// warp-level scans only (no block barrier inside the pass, 4 x float4 loads in flight per
// thread); three radix levels over the candidates give K*; the selected positions are
// marked in two shared-memory bitmaps (keys > K*, ties at K*) and written in position
// order with one block scan.  A row the fast path cannot settle (the sampled bound let
// fewer than k keys through, a candidate list overflowed, or a segment is longer than
// the bitmaps) gets -2 in its first output slot and is finished by the exact kernel.
constexpr int FT = 512;
constexpr int FCAP = 6144;
constexpr int FWORDS = 4096;  // bitmap words: segments up to 131072 positions

struct FastSmem {
  uint32_t cand_key[FCAP];
  int cand_pos[FCAP];
  uint32_t hist[2][2048];
  uint32_t ghist[2048];
  uint32_t gtb[FWORDS];   // positions with key > K*
  uint32_t tieb[FWORDS];  // positions with key == K*
  uint32_t warp_sums[32];
  uint32_t total, bin, above, ncand;
  uint32_t counts[2];
};

template <int C>
__global__ void __launch_bounds__(FT, 2) topk_fast_kernel(const TopkParams p) {
  constexpr int B = FT;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FastSmem& S = *reinterpret_cast<FastSmem*>(smem_raw);
  const int rank = (C > 1) ? (int)cg::this_cluster().block_rank() : 0;
  const int lane = threadIdx.x % 32;
  const long long row = p.row_begin + blockIdx.x / C;
  int lo = 0, hi = p.batch;
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
  int* out = p.indices + (row - p.row_begin) * k;
  const float* src = p.scores + (row - p.row_begin) * p.ld;
  if (vis <= k) {
    if (rank == 0)
      for (int j = threadIdx.x; j < k; j += B) out[j] = j < vis ? j : -1;
    return;
  }
  const int seg = ((vis + C - 1) / C + 3) & ~3;
  if (seg > FWORDS * 32) {  // uniform over the row
    if (rank == 0 && threadIdx.x == 0) out[0] = -2;
    return;
  }
  const int s_lo = min(rank * seg, vis), s_hi = min(s_lo + seg, vis);
  const int nwords = (s_hi - s_lo + 31) / 32;

  // ---------------------------------------------------------------- sampled bound T
  uint32_t T = 0;
  if (vis > C * (FCAP / 2)) {
    constexpr int NS = 2048, PER = NS / B;
    const float m = (float)k * (float)NS / (float)vis;
    const int r_low = min(NS, (int)ceilf(m + 3.f * sqrtf(m) + 8.f));
    uint32_t sk[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      const long long pos = ((2LL * (threadIdx.x + u * B) + 1) * vis) / (2LL * NS);
      sk[u] = float_order_key(__ldg(src + pos));
    }
    uint32_t sp = 0, sm = 0, rem = (uint32_t)r_low;
#pragma unroll 1
    for (int lv = 0; lv < 2; ++lv) {
      const int shift = lv == 0 ? 21 : 10;
      for (int j = threadIdx.x; j < 2048; j += B) S.ghist[j] = 0;
      __syncthreads();
#pragma unroll
      for (int u = 0; u < PER; ++u)
        if ((sk[u] & sm) == sp) atomicAdd(&S.ghist[(sk[u] >> shift) & 2047u], 1u);
      __syncthreads();
      find_bin<B, 2048>(S.ghist, rem, S.warp_sums, &S.total, &S.bin, &S.above);
      sp |= S.bin << shift;
      sm |= 2047u << shift;
      rem -= S.above;
    }
    T = sp;
  }

  // ---------------------------------------------------------------- streaming filter
  if (threadIdx.x == 0) S.ncand = 0;
  for (int w = threadIdx.x; w < nwords; w += B) {
    S.gtb[w] = 0;
    S.tieb[w] = 0;
  }
  __syncthreads();
  {
    constexpr int IT = 16;
    for (int start = s_lo; start < s_hi; start += B * IT) {
      const int s0 = start + threadIdx.x * IT;
      uint32_t key[IT];
      if (s0 + IT <= s_hi) {
        float4 x[IT / 4];
#pragma unroll
        for (int u = 0; u < IT / 4; ++u) x[u] = __ldg(reinterpret_cast<const float4*>(src + s0) + u);
#pragma unroll
        for (int u = 0; u < IT / 4; ++u) {
          key[4 * u + 0] = float_order_key(x[u].x);
          key[4 * u + 1] = float_order_key(x[u].y);
          key[4 * u + 2] = float_order_key(x[u].z);
          key[4 * u + 3] = float_order_key(x[u].w);
        }
      } else {
#pragma unroll
        for (int j = 0; j < IT; ++j) key[j] = (s0 + j < s_hi) ? float_order_key(__ldg(src + s0 + j)) : 0u;
      }
      uint32_t n = 0;
#pragma unroll
      for (int j = 0; j < IT; ++j) n += (s0 + j < s_hi && key[j] >= T);
      // warp-level exclusive scan and one shared counter bump per warp
      uint32_t x = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      uint32_t base = 0;
      if (lane == 31 && x) base = atomicAdd(&S.ncand, x);
      base = __shfl_sync(0xffffffffu, base, 31);
      uint32_t pos = base + x - n;
#pragma unroll
      for (int j = 0; j < IT; ++j) {
        if (s0 + j < s_hi && key[j] >= T) {
          if (pos < (uint32_t)FCAP) {
            S.cand_key[pos] = key[j];
            S.cand_pos[pos] = s0 + j;
          }
          ++pos;
        }
      }
    }
  }
  __syncthreads();
  const uint32_t cnt = S.ncand;
  // cluster-wide: enough keys passed, and every list fit
  if (threadIdx.x == 0) S.counts[0] = cnt;
  cluster_sync_all<C>();
  bool ok;
  {
    uint32_t tot = 0;
    bool fit = true;
    if constexpr (C == 1) {
      tot = S.counts[0];
      fit = tot <= (uint32_t)FCAP;
    } else {
      auto cl = cg::this_cluster();
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t c = *cl.map_shared_rank(&S.counts[0], r);
        tot += c;
        fit = fit && c <= (uint32_t)FCAP;
      }
    }
    ok = fit && tot >= (uint32_t)k;
  }
  cluster_sync_all<C>();
  if (!ok) {
    if (rank == 0 && threadIdx.x == 0) out[0] = -2;
    return;
  }
  const int ncand = (int)cnt;

  // ---------------------------------------------------------------- radix levels
  uint32_t remaining = (uint32_t)k, prefix = 0, pmask = 0;
#pragma unroll 1
  for (int level = 0; level < 3; ++level) {
    const int par = level & 1;
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const uint32_t bmask = level == 2 ? 1023u : 2047u;
    for (int j = threadIdx.x; j < 2048; j += B) S.hist[par][j] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < ncand; j += B) {
      const uint32_t kk = S.cand_key[j];
      if ((kk & pmask) == prefix) atomicAdd(&S.hist[par][(kk >> shift) & bmask], 1u);
    }
    cluster_sync_all<C>();
    const uint32_t* gh;
    if constexpr (C == 1) {
      gh = S.hist[par];
    } else {
      auto cl = cg::this_cluster();
      for (int j = threadIdx.x; j < 2048; j += B) {
        uint32_t t = 0;
#pragma unroll
        for (int r = 0; r < C; ++r) t += cl.map_shared_rank(&S.hist[par][0], r)[j];
        S.ghist[j] = t;
      }
      __syncthreads();
      gh = S.ghist;
    }
    if (level < 2)
      find_bin<B, 2048>(gh, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    else
      find_bin<B, 1024>(gh, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    prefix |= S.bin << shift;
    pmask |= bmask << shift;
    remaining -= S.above;
  }
  const uint32_t kstar = prefix;

  // ---------------------------------------------------------------- mark and write in order
  for (int j = threadIdx.x; j < ncand; j += B) {
    const uint32_t kk = S.cand_key[j];
    if (kk >= kstar) {
      const int r = S.cand_pos[j] - s_lo;
      atomicOr(kk > kstar ? &S.gtb[r >> 5] : &S.tieb[r >> 5], 1u << (r & 31));
    }
  }
  __syncthreads();
  const int wpt = (nwords + B - 1) / B;
  const int w0 = threadIdx.x * wpt, w1 = min(w0 + wpt, nwords);
  uint32_t my_gt = 0, my_tie = 0;
  for (int w = w0; w < w1; ++w) {
    my_gt += __popc(S.gtb[w]);
    my_tie += __popc(S.tieb[w]);
  }
  uint32_t gt_before = block_excl_scan<B>(my_gt, S.warp_sums, &S.total);
  const uint32_t tot_gt = S.total;
  __syncthreads();
  uint32_t tie_before = block_excl_scan<B>(my_tie, S.warp_sums, &S.total);
  const uint32_t tot_tie = S.total;
  if constexpr (C > 1) {
    if (threadIdx.x == 0) {
      S.counts[0] = tot_gt;
      S.counts[1] = tot_tie;
    }
    cluster_sync_all<C>();
    auto cl = cg::this_cluster();
    for (int r = 0; r < rank; ++r) {
      const uint32_t* rc = cl.map_shared_rank(&S.counts[0], r);
      gt_before += rc[0];
      tie_before += rc[1];
    }
  }
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = S.gtb[w] | S.tieb[w];
    const uint32_t gmask = S.gtb[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int pos = s_lo + w * 32 + bit;
      if (gmask & (1u << bit)) {
        out[gt_before + min(tie_before, remaining)] = pos;
        ++gt_before;
      } else {
        if (tie_before < remaining) out[gt_before + tie_before] = pos;
        ++tie_before;
      }
    }
  }
  if constexpr (C > 1) cg::this_cluster().sync();
}


// Visible positions of a row (bottom-right causal alignment).
__device__ __forceinline__ int row_visible(const TopkParams& p, long long row) {
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)p.cu_q[mid] <= row) lo = mid; else hi = mid;
  }
  const int i = (int)(row - p.cu_q[lo]);
  const int Lq = p.cu_q[lo + 1] - p.cu_q[lo];
  const int Lk = p.cu_k[lo + 1] - p.cu_k[lo];
  return min(max(i + Lk - Lq + 1, 0), Lk);
}

// ======================================================================================
// Helpers over a candidate list in shared memory (keys >= T, in position order).

// The exact k-th largest key K* among the n candidates, and how many keys equal to K* are
// taken, by radix levels over d = key - T.  The first level's 2048 bins span exactly
// [0, max d], so candidates that share their top key bits (scores in a narrow range) still
// spread over many bins instead of piling onto a few shared-memory counters.
template <int B>
__device__ void select_relative(const uint32_t* ckey, int n, uint32_t T, uint32_t k, uint32_t* hist,
                                uint32_t* warp_sums, uint32_t* total, uint32_t* bin, uint32_t* above,
                                uint32_t* dmax, uint32_t& kstar, uint32_t& remaining) {
  uint32_t dm = 0;
  for (int j = threadIdx.x; j < n; j += B) dm = max(dm, ckey[j] - T);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dm = max(dm, __shfl_xor_sync(0xffffffffu, dm, o));
  if (threadIdx.x == 0) *dmax = 0;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) atomicMax(dmax, dm);
  __syncthreads();
  const int nbits = 32 - __clz((int)*dmax);
  int shift = max(0, nbits - 11);
  uint32_t prefix = 0, pmask = 0, rem = k;
#pragma unroll 1
  while (true) {
    for (int j = threadIdx.x; j < 2048; j += B) hist[j] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += B) {
      const uint32_t d = ckey[j] - T;
      if ((d & pmask) == prefix) atomicAdd(&hist[(d >> shift) & 2047u], 1u);
    }
    __syncthreads();
    find_bin<B, 2048>(hist, rem, warp_sums, total, bin, above);
    prefix |= *bin << shift;
    pmask |= 2047u << shift;
    rem -= *above;
    if (shift == 0) break;
    shift = max(0, shift - 11);
  }
  kstar = T + prefix;
  remaining = rem;
}

// Writes the selected candidates (keys > K*, and the first `remaining` keys equal to K*)
// to out[0..k) in candidate order, which is position order.
template <int B>
__device__ void write_selected(const uint32_t* ckey, const int* cpos, int n, uint32_t kstar, uint32_t remaining,
                               int* out, uint32_t* warp_sums, uint32_t* total) {
  constexpr int IT = 4;  // tile totals <= B * IT fit the packed 16-bit fields
  static_assert(B * IT < 65536, "packed counts");
  uint32_t base_gt = 0, base_tie = 0;
  for (int start = 0; start < n; start += B * IT) {
    const int j0 = start + threadIdx.x * IT;
    uint32_t g_ = 0, e_ = 0;
#pragma unroll
    for (int j = 0; j < IT; ++j) {
      if (j0 + j < n) {
        g_ += ckey[j0 + j] > kstar;
        e_ += ckey[j0 + j] == kstar;
      }
    }
    const uint32_t excl = block_excl_scan<B>((g_ << 16) | e_, warp_sums, total);
    uint32_t gt_before = base_gt + (excl >> 16), eq_before = base_tie + (excl & 0xFFFFu);
#pragma unroll
    for (int j = 0; j < IT; ++j) {
      if (j0 + j >= n) break;
      const uint32_t kk = ckey[j0 + j];
      if (kk > kstar) {
        out[gt_before + min(eq_before, remaining)] = cpos[j0 + j];
        ++gt_before;
      } else if (kk == kstar) {
        if (eq_before < remaining) out[gt_before + eq_before] = cpos[j0 + j];
        ++eq_before;
      }
    }
    base_gt += *total >> 16;
    base_tie += *total & 0xFFFFu;
    __syncthreads();
  }
}

// A fixed strided sample of NS positions of a row (PER keys per thread), and from it the
// r_low-th largest sampled key to 22 bits: a lower bound on the row's k-th largest key
// with a margin of ~3 sigma + 8 sampled keys.  Every block that samples the same row gets
// the same value.
constexpr int SAMPLE_N = 2048;

template <int B>
__device__ __forceinline__ void load_sample(const float* src, int vis, uint32_t* sk) {
#pragma unroll
  for (int u = 0; u < SAMPLE_N / B; ++u) {
    const long long pos = ((2LL * (threadIdx.x + u * B) + 1) * vis) / (2LL * SAMPLE_N);
    sk[u] = float_order_key(__ldg(src + pos));
  }
}

template <int B>
__device__ uint32_t bound_from_sample(const uint32_t* sk, int vis, int k, uint32_t* hist, uint32_t* warp_sums,
                                      uint32_t* total, uint32_t* bin, uint32_t* above) {
  constexpr int PER = SAMPLE_N / B;
  static_assert(SAMPLE_N % B == 0, "samples per thread");
  const float m = (float)k * (float)SAMPLE_N / (float)vis;
  const int r_low = min(SAMPLE_N, (int)ceilf(m + 3.f * sqrtf(m) + 8.f));
  uint32_t sp = 0, sm = 0, rem = (uint32_t)r_low;
#pragma unroll 1
  for (int lv = 0; lv < 2; ++lv) {
    const int shift = lv == 0 ? 21 : 10;
    for (int j = threadIdx.x; j < 2048; j += B) hist[j] = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      // samples of a row often share their top bits: one counter update per distinct bin
      // and warp instead of one per sample
      const bool act = (sk[u] & sm) == sp;
      const uint32_t b = act ? (sk[u] >> shift) & 2047u : 0xFFFFFFFFu;
      const uint32_t peers = __match_any_sync(0xffffffffu, b);
      if (act && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[b], (uint32_t)__popc(peers));
    }
    __syncthreads();
    find_bin<B, 2048>(hist, rem, warp_sums, total, bin, above);
    sp |= *bin << shift;
    sm |= 2047u << shift;
    rem -= *above;
  }
  return sp;
}

template <int B>
__device__ uint32_t sampled_bound(const float* src, int vis, int k, uint32_t* hist, uint32_t* warp_sums,
                                  uint32_t* total, uint32_t* bin, uint32_t* above) {
  uint32_t sk[SAMPLE_N / B];
  load_sample<B>(src, vis, sk);
  return bound_from_sample<B>(sk, vis, k, hist, warp_sums, total, bin, above);
}

// ======================================================================================
// Few long rows (decode: a handful of sequences with 10^5 cached positions each).  A row
// goes to a cluster of C blocks of 512 threads; the block reads its segment once with 16
// coalesced float4 loads per thread (all in flight at once) and hands every thread 64
// consecutive scores in registers through a swizzled shared-memory transpose.
//   1. While those loads fly, every block takes the same strided sample of 2048 positions
//      and, by two radix levels, the r_low-th largest sampled key T (a lower bound on the
//      k-th largest key, with a safety margin).
//   2. Keys >= T are counted in registers (no atomics); the blocks exchange their counts.
//      If they add up to at least k and fit rank 0's candidate list, every block writes
//      its candidates, in position order, into rank 0's shared memory.  Rank 0 then finds
//      the exact k-th key K* by radix levels over (key - T), whose 2048 bins span exactly
//      the candidates' range, and writes the selected positions in order.
//   3. Otherwise (an unlucky sample, or huge ties) all blocks run three radix levels
//      (11 + 11 + 10 key bits) over the register-resident keys, each level's histogram
//      summed over the cluster through distributed shared memory, and write in order
//      from the per-block counts.
// The sample only decides how the exact K* is found, never which positions are selected.
// Rows up to C x 32768 positions (C <= 8, the portable cluster size).
constexpr int RT = 512;           // threads per block
constexpr int RKEYS = 64;         // keys per thread
constexpr int RSEG = RT * RKEYS;  // positions per block
constexpr int RCAP = 16384;       // candidates rank 0 can hold

struct RegsSmem {
  union {
    float4 seg[RSEG / 4];  // the block's scores, swizzled 16-byte chunks (load transpose)
    struct {
      uint32_t cand_key[RCAP];  // rank 0: the row's candidates in position order
      int cand_pos[RCAP];
    };
  };
  uint32_t hist[2][2048];  // per level parity (remote blocks read them)
  uint32_t ghist[2048];    // cluster-wide sum
  uint32_t warp_sums[32];
  uint32_t total, bin, above, dmax;
  uint32_t counts[2];
};

template <int C>
__global__ void __launch_bounds__(RT, 1) topk_regs_kernel(const TopkParams p) {
  constexpr int B = RT;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RegsSmem& S = *reinterpret_cast<RegsSmem*>(smem_raw);
  auto cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const long long row = p.row_begin + blockIdx.x / C;
  int lo = 0, hi = p.batch;
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
  int* out = p.indices + (row - p.row_begin) * k;
  const float* src = p.scores + (row - p.row_begin) * p.ld;
  if (vis <= k) {  // uniform over the cluster
    if (rank == 0)
      for (int j = threadIdx.x; j < k; j += B) out[j] = j < vis ? j : -1;
    return;
  }
  // block segment [s_lo, s_hi) (4-aligned starts); this thread: [t_lo, t_lo + RKEYS)
  const int seg = ((vis + C - 1) / C + 3) & ~3;
  const int s_lo = min(rank * seg, vis), s_hi = min(s_lo + seg, vis);
  const int t_lo = s_lo + threadIdx.x * RKEYS;
  const int nvalid = max(0, min(RKEYS, s_hi - t_lo));  // keys [0, nvalid) of this thread are real
  // coalesced loads: 16-byte chunk q = u * B + tid of the segment, stored at chunk
  // q ^ ((q >> 4) & 7) so that both this store and the per-thread reads below (16
  // consecutive chunks of one thread) are free of bank conflicts
  {
    float4 x[RKEYS / 4];
#pragma unroll
    for (int u = 0; u < RKEYS / 4; ++u) {
      const int q = u * B + threadIdx.x;
      x[u] = (s_lo + 4 * q < s_hi) ? __ldg(reinterpret_cast<const float4*>(src + s_lo) + q)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < RKEYS / 4; ++u) {
      const int q = u * B + threadIdx.x;
      S.seg[q ^ ((q >> 4) & 7)] = x[u];
    }
  }

  // ---------------------------------------------------------------- 1. sampled bound T
  const uint32_t T = sampled_bound<B>(src, vis, k, S.ghist, S.warp_sums, &S.total, &S.bin, &S.above);
  __syncthreads();  // the segment is in shared memory
  uint32_t key[RKEYS];
#pragma unroll
  for (int u = 0; u < RKEYS / 4; ++u) {
    const int q = threadIdx.x * (RKEYS / 4) + u;
    const float4 x = S.seg[q ^ ((q >> 4) & 7)];
    key[4 * u + 0] = float_order_key(x.x);
    key[4 * u + 1] = float_order_key(x.y);
    key[4 * u + 2] = float_order_key(x.z);
    key[4 * u + 3] = float_order_key(x.w);
  }

  // ---------------------------------------------------------------- 2. candidates >= T
  uint32_t n_c = 0;
#pragma unroll
  for (int j = 0; j < RKEYS; ++j) n_c += (j < nvalid && key[j] >= T);
  const uint32_t c_before = block_excl_scan<B>(n_c, S.warp_sums, &S.total);
  if (threadIdx.x == 0) S.counts[0] = S.total;
  cl.sync();
  uint32_t base = 0, N = 0;
  bool fits = true;
#pragma unroll
  for (int r = 0; r < C; ++r) {
    const uint32_t c = *cl.map_shared_rank(&S.counts[0], r);
    if (r < rank) base += c;
    N += c;
  }
  fits = N >= (uint32_t)k && N <= (uint32_t)RCAP;
  if (fits) {
    uint32_t* rk = cl.map_shared_rank(&S.cand_key[0], 0);
    int* rp = cl.map_shared_rank(&S.cand_pos[0], 0);
    uint32_t pos = base + c_before;
#pragma unroll
    for (int j = 0; j < RKEYS; ++j) {
      if (j < nvalid && key[j] >= T) {
        rk[pos] = key[j];
        rp[pos] = t_lo + j;
        ++pos;
      }
    }
    cl.sync();  // the candidates have landed in rank 0; nothing else is read remotely
    if (rank != 0) return;
    uint32_t kstar, remaining;
    select_relative<B>(S.cand_key, (int)N, T, (uint32_t)k, S.ghist, S.warp_sums, &S.total, &S.bin, &S.above, &S.dmax,
                       kstar, remaining);
    write_selected<B>(S.cand_key, S.cand_pos, (int)N, kstar, remaining, out, S.warp_sums, &S.total);
    return;
  }

  // ---------------------------------------------------------------- 3. exact levels over the registers
  uint32_t remaining = (uint32_t)k, prefix = 0, pmask = 0;
#pragma unroll 1
  for (int level = 0; level < 3; ++level) {
    const int par = level & 1;
    const int shift = level == 0 ? 21 : (level == 1 ? 10 : 0);
    const uint32_t bmask = level == 2 ? 1023u : 2047u;
    for (int j = threadIdx.x; j < 2048; j += B) S.hist[par][j] = 0;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < RKEYS; ++j)
      if (j < nvalid && (key[j] & pmask) == prefix) atomicAdd(&S.hist[par][(key[j] >> shift) & bmask], 1u);
    cl.sync();
    const int nb = level == 2 ? 1024 : 2048;
    for (int j = threadIdx.x; j < nb; j += B) {
      uint32_t t = 0;
#pragma unroll
      for (int r = 0; r < C; ++r) t += cl.map_shared_rank(&S.hist[par][0], r)[j];
      S.ghist[j] = t;
    }
    __syncthreads();
    if (level < 2)
      find_bin<B, 2048>(S.ghist, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    else
      find_bin<B, 1024>(S.ghist, remaining, S.warp_sums, &S.total, &S.bin, &S.above);
    prefix |= S.bin << shift;
    pmask |= bmask << shift;
    remaining -= S.above;
  }
  const uint32_t kstar = prefix;
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < RKEYS; ++j) {
    n_gt += (j < nvalid && key[j] > kstar);
    n_eq += (j < nvalid && key[j] == kstar);
  }
  // per-thread counts <= 64 and block totals <= RSEG = 32768 fit the packed 16-bit fields
  const uint32_t excl = block_excl_scan<B>((n_gt << 16) | n_eq, S.warp_sums, &S.total);
  if (threadIdx.x == 0) {
    S.counts[0] = S.total >> 16;
    S.counts[1] = S.total & 0xFFFFu;
  }
  cl.sync();
  uint32_t gt_before = excl >> 16, eq_before = excl & 0xFFFFu;
  for (int r = 0; r < rank; ++r) {
    const uint32_t* rc = cl.map_shared_rank(&S.counts[0], r);
    gt_before += rc[0];
    eq_before += rc[1];
  }
#pragma unroll
  for (int j = 0; j < RKEYS; ++j) {
    if (j < nvalid) {
      if (key[j] > kstar) {
        out[gt_before + min(eq_before, remaining)] = t_lo + j;
        ++gt_before;
      } else if (key[j] == kstar) {
        if (eq_before < remaining) out[gt_before + eq_before] = t_lo + j;
        ++eq_before;
      }
    }
  }
  cl.sync();  // no block may leave while another still reads its shared memory
}

// ======================================================================================
// Many rows (prefill chunks: thousands of rows of up to ~10^5 positions).  One 256-thread
// block per row, four blocks per SM, so the latency-bound steps of some rows overlap the
// streaming of others:
//   1. the row's sampled bound T (a strided sample of 2048 scores);
//   2. one streaming pass over the row in tiles of 4096 positions (16 consecutive per
//      thread, the next tile's loads issued before this tile is compacted): keys >= T are
//      appended to a shared-memory list by a block scan per tile, so the list is in
//      position order;
//   3. the exact K* by radix levels over (key - T) on the list, and the ordered output.
// A row whose list would overflow, or holds fewer than k keys (an unlucky sample), gets -2
// in its first output slot and is finished by the exact kernel.
constexpr int ST_T = 256;
constexpr int ST_ITEMS = 16;
constexpr int ST_TILE = ST_T * ST_ITEMS;
constexpr int ST_CAP = 4096;

struct StreamSmem {
  uint32_t cand_key[ST_CAP];
  int cand_pos[ST_CAP];
  uint32_t hist[2048];
  uint32_t warp_sums[32];
  uint32_t total, bin, above, dmax;
};

__global__ void __launch_bounds__(ST_T, 4) topk_stream_kernel(const TopkParams p) {
  constexpr int B = ST_T;
  __shared__ StreamSmem S;
  const long long row = p.row_begin + blockIdx.x;
  const int vis = row_visible(p, row);
  const int k = p.k;
  int* out = p.indices + (row - p.row_begin) * k;
  const float* src = p.scores + (row - p.row_begin) * p.ld;
  if (vis <= k) {
    for (int j = threadIdx.x; j < k; j += B) out[j] = j < vis ? j : -1;
    return;
  }
  // loads ST_ITEMS scores of positions [s0, s0 + ST_ITEMS) (s0 4-aligned), 0 past the row
  auto load = [&](int s0, float4* x) {
#pragma unroll
    for (int u = 0; u < ST_ITEMS / 4; ++u)
      x[u] = (s0 + 4 * u < vis) ? __ldg(reinterpret_cast<const float4*>(src + s0) + u) : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  float4 cur[ST_ITEMS / 4];
  load(threadIdx.x * ST_ITEMS, cur);  // first tile in flight during the sample
  const uint32_t T = sampled_bound<B>(src, vis, k, S.hist, S.warp_sums, &S.total, &S.bin, &S.above);

  uint32_t base = 0;
  for (int tile = 0; tile < vis; tile += ST_TILE) {
    const int s0 = tile + threadIdx.x * ST_ITEMS;
    float4 nxt[ST_ITEMS / 4];
    load(s0 + ST_TILE, nxt);
    uint32_t key[ST_ITEMS];
#pragma unroll
    for (int u = 0; u < ST_ITEMS / 4; ++u) {
      key[4 * u + 0] = float_order_key(cur[u].x);
      key[4 * u + 1] = float_order_key(cur[u].y);
      key[4 * u + 2] = float_order_key(cur[u].z);
      key[4 * u + 3] = float_order_key(cur[u].w);
    }
    uint32_t n = 0;
#pragma unroll
    for (int j = 0; j < ST_ITEMS; ++j) n += (s0 + j < vis && key[j] >= T);
    uint32_t pos = base + block_excl_scan<B>(n, S.warp_sums, &S.total);
#pragma unroll
    for (int j = 0; j < ST_ITEMS; ++j) {
      if (s0 + j < vis && key[j] >= T) {
        if (pos < (uint32_t)ST_CAP) {
          S.cand_key[pos] = key[j];
          S.cand_pos[pos] = s0 + j;
        }
        ++pos;
      }
    }
    base += S.total;
#pragma unroll
    for (int u = 0; u < ST_ITEMS / 4; ++u) cur[u] = nxt[u];
    // (S.total is rewritten only after the next scan's first barrier)
  }
  __syncthreads();
  if (base < (uint32_t)k || base > (uint32_t)ST_CAP) {
    if (threadIdx.x == 0) out[0] = -2;
    return;
  }
  uint32_t kstar, remaining;
  select_relative<B>(S.cand_key, (int)base, T, (uint32_t)k, S.hist, S.warp_sums, &S.total, &S.bin, &S.above, &S.dmax,
                     kstar, remaining);
  write_selected<B>(S.cand_key, S.cand_pos, (int)base, kstar, remaining, out, S.warp_sums, &S.total);
}

// ======================================================================================
// Few long rows with a caller workspace (the decode shape: 16 sequences x 262144 cached
// positions).  Three launches, no clusters, so every SM takes part however the GPCs are
// filled:
//   0. row bound: one block per row takes the row's sampled bound T.
//   1. segment filter: one 256-thread block per (row, 8192-position segment).  The block
//      reads its segment once (coalesced float4 loads, handed to the threads as 32
//      consecutive scores each through a swizzled shared-memory transpose) and writes its
//      keys >= T, in position order, to the workspace with their count.
//   2. row select: one 1024-thread block per row gathers the segments' candidates in
//      order, finds the exact K* by radix levels over (key - T) and writes the selected
//      positions.  A row whose candidates are too few (an unlucky sample), overflow a
//      segment or the block's list (huge ties) is selected by the exact method from the
//      scores instead.  Either way the result is the exact top-k.
constexpr int SF_T = 256;                 // threads of a segment-filter block
constexpr int SF_SEG = 8192;              // positions per segment
constexpr int SF_KEYS = SF_SEG / SF_T;    // keys per thread
constexpr int SF_CAP = 1024;              // candidates kept per segment
constexpr int SF_MAX_BLOCKS = 1024;       // rows x segments beyond which this path is not used

struct TopkWs {
  uint32_t* thr;  // [rows] sampled bound T of each row (written for rows with vis > k)
  uint32_t* cnt;  // [rows, nseg] candidates of each segment (may exceed SF_CAP: overflow)
  uint2* cand;    // [rows, nseg, SF_CAP] (key, position)
  int nseg;
};

struct SegFilterSmem {
  float4 seg[SF_SEG / 4];
  uint32_t ghist[2048];
  uint32_t warp_sums[32];
  uint32_t total, bin, above;
};


// The sampled bound T of each row, once per row (a sample read by every filter block of
// the row would hit the same L2 sectors from all of them at once).
__global__ void __launch_bounds__(SF_T) topk_rowbound_kernel(const TopkParams p, const TopkWs ws) {
  constexpr int B = SF_T;
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t total, bin, above;
  const long long rr = blockIdx.x;
  const int vis = row_visible(p, p.row_begin + rr);
  if (vis <= p.k) return;
  const uint32_t T = sampled_bound<B>(p.scores + rr * p.ld, vis, p.k, hist, warp_sums, &total, &bin, &above);
  if (threadIdx.x == 0) ws.thr[rr] = T;
}

__global__ void __launch_bounds__(SF_T, 4) topk_segfilter_kernel(const TopkParams p, const TopkWs ws) {
  constexpr int B = SF_T;
  pdl_wait();
  __shared__ SegFilterSmem S;
  const long long rr = blockIdx.x / ws.nseg;
  const int sg = blockIdx.x % ws.nseg;
  const long long row = p.row_begin + rr;
  const int vis = row_visible(p, row);
  if (vis <= p.k) return;  // the row-select block handles such rows without the workspace
  uint32_t* cnt = ws.cnt + rr * ws.nseg + sg;
  const int s_lo = sg * SF_SEG;
  if (s_lo >= vis) {
    if (threadIdx.x == 0) *cnt = 0;
    return;
  }
  const int s_hi = min(s_lo + SF_SEG, vis);
  const float* src = p.scores + rr * p.ld;
  {
    // chunk q = u * B + tid, stored at q ^ ((q >> 3) & 7): conflict-free here and for the
    // per-thread reads of 8 consecutive chunks below
    float4 x[SF_KEYS / 4];
#pragma unroll
    for (int u = 0; u < SF_KEYS / 4; ++u) {
      const int q = u * B + threadIdx.x;
      x[u] = (s_lo + 4 * q < s_hi) ? __ldg(reinterpret_cast<const float4*>(src + s_lo) + q)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < SF_KEYS / 4; ++u) {
      const int q = u * B + threadIdx.x;
      S.seg[q ^ ((q >> 3) & 7)] = x[u];
    }
  }
  const uint32_t T = ws.thr[rr];
  __syncthreads();  // the segment is in shared memory
  const int t_lo = s_lo + threadIdx.x * SF_KEYS;
  const int nvalid = max(0, min(SF_KEYS, s_hi - t_lo));
  // this thread's keys are re-read from shared memory (16-byte reads) in each of the two passes
  auto chunk_at = [&](int u) -> float4 {
    const int q = threadIdx.x * (SF_KEYS / 4) + u;
    return S.seg[q ^ ((q >> 3) & 7)];
  };
  uint32_t n = 0;
#pragma unroll
  for (int u = 0; u < SF_KEYS / 4; ++u) {
    const float4 x = chunk_at(u);
    const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) n += (4 * u + e < nvalid && float_order_key(v[e]) >= T);
  }
  uint32_t pos = block_excl_scan<B>(n, S.warp_sums, &S.total);
  uint2* dst = ws.cand + (rr * ws.nseg + sg) * SF_CAP;
#pragma unroll
  for (int u = 0; u < SF_KEYS / 4; ++u) {
    const float4 x = chunk_at(u);
    const float v[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t kj = float_order_key(v[e]);
      if (4 * u + e < nvalid && kj >= T) {
        if (pos < (uint32_t)SF_CAP) dst[pos] = make_uint2(kj, (uint32_t)(t_lo + 4 * u + e));
        ++pos;
      }
    }
  }
  if (threadIdx.x == 0) *cnt = S.total;
  pdl_trigger();  // late: the next kernel's blocks would take this one's SM slots
}

__global__ void __launch_bounds__(TOPK_THREADS) topk_rowselect_kernel(const TopkParams p, const TopkWs ws) {
  constexpr int B = TOPK_THREADS;
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& S = *reinterpret_cast<TopkSmem*>(smem_raw);
  const long long rr = blockIdx.x;
  const long long row = p.row_begin + rr;
  const int vis = row_visible(p, row);
  const int k = p.k;
  int* out = p.indices + rr * k;
  if (vis <= k) {
    for (int j = threadIdx.x; j < k; j += B) out[j] = j < vis ? j : -1;
    return;
  }
  const int nseg = (vis + SF_SEG - 1) / SF_SEG;  // <= ws.nseg <= B (host-checked)
  const uint32_t c = threadIdx.x < nseg ? ws.cnt[rr * ws.nseg + threadIdx.x] : 0u;
  const bool overflow = __syncthreads_or(c > (uint32_t)SF_CAP) != 0;
  const uint32_t base = block_excl_scan<B>(c, S.warp_sums, &S.total);
  const uint32_t N = S.total;
  if (!overflow && N >= (uint32_t)k && N <= (uint32_t)TOPK_CAP) {
    if (threadIdx.x < nseg) S.ghist[threadIdx.x] = base;  // segment start in the list
    __syncthreads();
    // warp w gathers segments w, w + 32, ...: coalesced, and in position order overall
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    for (int sgi = warp; sgi < nseg; sgi += B / 32) {
      const uint2* srcc = ws.cand + (rr * ws.nseg + sgi) * SF_CAP;
      const uint32_t b0 = S.ghist[sgi];
      const uint32_t cn = ws.cnt[rr * ws.nseg + sgi];
      for (uint32_t j = lane; j < cn; j += 32) {
        const uint2 e = srcc[j];
        S.cand_key[b0 + j] = e.x;
        S.cand_pos[b0 + j] = (int)e.y;
      }
    }
    __syncthreads();
    uint32_t kstar, remaining;
    select_relative<B>(S.cand_key, (int)N, ws.thr[rr], (uint32_t)k, S.hist[0], S.warp_sums, &S.total, &S.bin,
                       &S.above, &S.dmax, kstar, remaining);
    write_selected<B>(S.cand_key, S.cand_pos, (int)N, kstar, remaining, out, S.warp_sums, &S.total);
    return;
  }
  __syncthreads();  // S.total and S.warp_sums are reused by the exact method
  exact_row_select<1>(p, S, row);
}

}  // namespace dsa

namespace dsa_host {

template <typename Kern>
static int launch_cluster(Kern kern, const dsa::TopkParams& p, long long rows, int C, int threads, int smem,
                          DeviceFlag& attr_done, cudaStream_t stream) {
  if (!attr_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * C), 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = C > 1 ? 1 : 0;
  if (const cudaError_t e_ = cudaLaunchKernelEx(&cfg, kern, p); e_ != cudaSuccess) return cuda_fail(e_);
  return last_launch_status();
}

template <int C>
static int topk_launch_c(dsa::TopkParams p, long long rows, cudaStream_t stream) {
  static DeviceFlag fast_done, exact_done;
  p.only_marked = 0;
  int st = launch_cluster(dsa::topk_fast_kernel<C>, p, rows, C, dsa::FT, (int)sizeof(dsa::FastSmem), fast_done,
                          stream);
  if (st != DSA_OK) return st;
  p.only_marked = 1;  // rows the fast path left marked
  return launch_cluster(dsa::topk_kernel<C>, p, rows, C, dsa::TOPK_THREADS, (int)sizeof(dsa::TopkSmem), exact_done,
                        stream);
}

template <int C>
static int topk_regs_launch(const dsa::TopkParams& p, long long rows, cudaStream_t stream) {
  static_assert(C <= 8, "portable cluster sizes only");
  static DeviceFlag attr_done;
  if (!attr_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_regs_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)sizeof(dsa::RegsSmem));
    if (e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * C), 1, 1);
  cfg.blockDim = dim3(dsa::RT, 1, 1);
  cfg.dynamicSmemBytes = sizeof(dsa::RegsSmem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (const cudaError_t e_ = cudaLaunchKernelEx(&cfg, dsa::topk_regs_kernel<C>, p); e_ != cudaSuccess)
    return cuda_fail(e_);
  return last_launch_status();
}

// The exact selection of the rows of [p.row_begin, p.row_begin + rows) whose first index
// slot holds -2, from the score rows in p.scores; the other rows are left as they are.
static int topk_marked_rows_launch(dsa::TopkParams p, long long rows, cudaStream_t stream) {
  static DeviceFlag exact_done;
  p.only_marked = 1;
  if (!exact_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_marked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                (int)sizeof(dsa::TopkSmem));
    if (e_ != cudaSuccess) return cuda_fail(e_);
    exact_done = true;
  }
  const long long grid = std::max((rows + dsa::TOPK_THREADS - 1) / dsa::TOPK_THREADS, std::min(rows, (long long)sm_count()));
  dsa::topk_marked_kernel<<<(unsigned)grid, dsa::TOPK_THREADS, sizeof(dsa::TopkSmem), stream>>>(p, rows);
  return last_launch_status();
}

// One block per row with the streaming kernel, then the exact kernel for rows it marked.
static int topk_stream_launch(dsa::TopkParams p, long long rows, cudaStream_t stream) {
  static DeviceFlag attr_done;
  if (!attr_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_stream_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  p.only_marked = 0;
  dsa::topk_stream_kernel<<<(unsigned)rows, dsa::ST_T, 0, stream>>>(p);
  if (const int st = last_launch_status(); st != DSA_OK) return st;
  return topk_marked_rows_launch(p, rows, stream);
}

// Exact top-k of the rows of [row_begin, row_end) that an earlier pass marked with -2 in
// their first index slot (indices points at row row_begin's slots).
int topk_marked_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                       long long row_begin, long long row_end, int k, int* indices, int* flag_reset,
                       cudaStream_t stream) {
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
  p.only_marked = 1;
  p.flag_reset = flag_reset;
  return topk_marked_rows_launch(p, rows, stream);
}

// Workspace of the two-launch path for `rows` rows of up to max_vis positions; 0 where
// that path is not used (many rows, short rows or rows beyond its segment count).
size_t topk_ws_bytes(long long rows, long long max_vis) {
  if (rows <= 0 || max_vis <= 32768) return 0;
  const long long nseg = (max_vis + dsa::SF_SEG - 1) / dsa::SF_SEG;
  if (nseg > dsa::TOPK_THREADS || rows * nseg > dsa::SF_MAX_BLOCKS) return 0;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  return up((size_t)rows * 4) + up((size_t)(rows * nseg) * 4) + up((size_t)(rows * nseg) * dsa::SF_CAP * 8);
}

static int topk_two_launch(const dsa::TopkParams& p, long long rows, long long max_vis, void* ws_ptr,
                           cudaStream_t stream) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  dsa::TopkWs ws;
  ws.nseg = (int)((max_vis + dsa::SF_SEG - 1) / dsa::SF_SEG);
  uint8_t* w = static_cast<uint8_t*>(ws_ptr);
  ws.thr = reinterpret_cast<uint32_t*>(w);
  w += up((size_t)rows * 4);
  ws.cnt = reinterpret_cast<uint32_t*>(w);
  w += up((size_t)(rows * ws.nseg) * 4);
  ws.cand = reinterpret_cast<uint2*>(w);
  static DeviceFlag attr_done;
  if (!attr_done) {
    // four filter blocks per SM need the largest shared-memory carveout
    cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_segfilter_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                          100);
    if (e_ == cudaSuccess)
      e_ = cudaFuncSetAttribute(dsa::topk_rowselect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)sizeof(dsa::TopkSmem));
    if (e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  // the second and third launches overlap their launch latency with the previous kernel's
  // tail (programmatic dependent launch)
  if (const int st = launch_pdl(false, dsa::topk_rowbound_kernel, dim3((unsigned)rows), dim3(dsa::SF_T), 0, stream, p, ws);
      st != DSA_OK)
    return st;
  if (const int st = launch_pdl(true, dsa::topk_segfilter_kernel, dim3((unsigned)(rows * ws.nseg)), dim3(dsa::SF_T), 0,
                                stream, p, ws);
      st != DSA_OK)
    return st;
  return launch_pdl(true, dsa::topk_rowselect_kernel, dim3((unsigned)rows), dim3(dsa::TOPK_THREADS), sizeof(dsa::TopkSmem),
                    stream, p, ws);
}

int topk_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                long long row_begin, long long row_end, int k, int* indices, int max_vis, void* ws,
                size_t ws_bytes, cudaStream_t stream) {
  const long long rows = row_end - row_begin;
  if (rows <= 0) return DSA_OK;
  if (rows > 0x7FFFFFFFLL / 16) return DSA_ERR_UNSUPPORTED;
  dsa::TopkParams p;
  p.scores = scores;
  p.ld = ld;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.row_begin = row_begin;
  p.k = k;
  p.indices = indices;
  p.only_marked = 0;
  const int sms = sm_count();
  // few long rows with a workspace: segment filter + row select
  if (const size_t need = topk_ws_bytes(rows, max_vis); need > 0 && ws != nullptr && ws_bytes >= need)
    return topk_two_launch(p, rows, max_vis, ws, stream);
  // few long rows: one cluster per row with the row held in registers, while that takes
  // at most two waves of one block per SM
  if (max_vis > 32768) {
    int C = 4;
    while (C < 8 && (long long)C * dsa::RSEG < (long long)max_vis) C *= 2;
    if ((long long)C * dsa::RSEG >= (long long)max_vis && rows * C <= 2LL * sms)
      return C == 4 ? topk_regs_launch<4>(p, rows, stream) : topk_regs_launch<8>(p, rows, stream);
  }
  // a cluster per row when the rows are long and few enough blocks would be busy otherwise
  int C = 1;
  while (C < 8 && (long long)rows * C < 2LL * sms && (long long)max_vis > 16384LL * C) C *= 2;
  switch (C) {
    case 1: return topk_stream_launch(p, rows, stream);
    case 2: return topk_launch_c<2>(p, rows, stream);
    case 4: return topk_launch_c<4>(p, rows, stream);
    default: return topk_launch_c<8>(p, rows, stream);
  }
}

}  // namespace dsa_host
