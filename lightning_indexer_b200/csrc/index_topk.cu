// Fused lightning indexer -> deterministic top-k (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1 (the indexer scans
// every visible position and each token keeps its 2048 best) and section 8 (the top-k
// must be deterministic).  The separate path writes every score of a row chunk to an fp32
// scratch and reads it back to select (34 GB each way at 128K context); here the indexer
// keeps only the scores that can still be among a row's k largest.
//
// Two phases:
//   A. over all rows, in as few launches as the scratch allows:
//      1. sampled scores: the CTA-pair indexer over every S-th indexer key (S a power of two
//         chosen so that a full row has at most about 1024 samples), about 1/S of the work;
//      2. bound: per row (one warp), the c-th largest sampled score cut to 22 key bits, by
//         bisection on the order key; c = m + 3 sqrt(m) + 8 with m = k / S, the number of
//         samples expected at or above the row's k-th largest score.  Rows with at most
//         `cap` visible positions get no bound (every position is a candidate).  The bound
//         and the row's candidate count live in the row's own output slots (k-1 and k-2)
//         until the row is selected.
//   B. per row chunk:
//      3. fused indexer: every score whose order key reaches the row's bound is appended to
//         the row's candidate list as (key, position); no score matrix is written;
//      4. select: per row, one histogram of the candidates' keys relative to the bound
//         locates the bin of the k-th largest key; higher bins are selected outright and
//         the few keys of that bin are ranked exactly by (key descending, position
//         ascending); a bitmap over the row and a block scan write the positions in
//         ascending order, whatever order the candidates arrived in.  A row with fewer
//         than k candidates (an unlucky sample), more than `cap`, or more than 256 keys in
//         the boundary bin (huge ties) is marked -2 and raises the chunk's repair flag;
//      5. repair: only if the flag is raised, the indexer writes the full score rows of the
//         marked rows' blocks to the scratch and the exact top-k selects them (and clears
//         the flag).
// Every candidate list holds exactly the positions whose key reaches the bound, and the
// bound only decides how many positions are kept, never which of them are selected: the
// result is the exact top-k of the rows' scores, bit for bit the one the separate path
// returns on the same scores.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct FusedTopkParams {
  const float* samples;  // [rows, ld_s] sampled scores of the rows from row_begin on
  long long ld_s;
  int S;                 // key stride of the samples
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin;   // first row of the launch
  long long rows;
  int k;
  int cap;               // candidates kept per row
  uint32_t* thr;         // bound (order key) of row rr at thr[rr * state_ld]
  uint32_t* cnt;         // candidates appended to row rr at cnt[rr * state_ld]
  long long state_ld;
  int* flag;             // set when a row needs the repair pass
  const uint2* cand;     // [rows, cap] (order key, position)
  int* indices;          // [rows, k] output of the launch's rows
};

// Visible positions and first packed key of a row (bottom-right causal alignment).
__device__ __forceinline__ void fused_row_geometry(const FusedTopkParams& p, long long row, int& vis, int& kg) {
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)p.cu_q[mid] <= row) lo = mid; else hi = mid;
  }
  kg = p.cu_k[lo];
  vis = causal_vis((int)(row - p.cu_q[lo]), p.cu_q[lo + 1] - p.cu_q[lo], p.cu_k[lo + 1] - kg);
}

constexpr int SB_WARPS = 8;  // rows (one warp each) per bound block
constexpr int SB_KPL = 40;   // sampled scores per lane: rows of up to 1280 samples

// Step 2: one warp per row.  Also zeroes the row's candidate count.
__global__ void __launch_bounds__(SB_WARPS * 32) topk_sample_bound_kernel(const FusedTopkParams p) {
  const long long rr = (long long)blockIdx.x * SB_WARPS + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (rr >= p.rows) return;
  int vis, kg;
  fused_row_geometry(p, p.row_begin + rr, vis, kg);
  if (lane == 0) p.cnt[rr * p.state_ld] = 0u;
  const long long S = p.S;
  const int ns = (int)((kg + (long long)vis + S - 1) / S - (kg + S - 1) / S);  // sampled positions
  const float m = (float)p.k / (float)S;
  const int c = (int)ceilf(m + 3.f * sqrtf(m) + 8.f);
  if (vis <= p.cap || c >= ns) {  // every visible position is a candidate
    if (lane == 0) p.thr[rr * p.state_ld] = 0u;
    return;
  }
  const float* src = p.samples + rr * p.ld_s;
  uint32_t key[SB_KPL];
#pragma unroll
  for (int u = 0; u < SB_KPL; ++u) {
    const int j = u * 32 + lane;
    key[u] = j < ns ? float_order_key(__ldg(src + j)) : 0u;  // 0: below every tested bound
  }
  // the largest T with its low 10 bits clear such that at least c sampled keys are >= T,
  // i.e. the c-th largest sampled key cut to 22 bits
  uint32_t T = 0;
#pragma unroll 1
  for (int b = 31; b >= 10; --b) {
    const uint32_t t = T | (1u << b);
    uint32_t n = 0;
#pragma unroll
    for (int u = 0; u < SB_KPL; ++u) n += key[u] >= t;
    if (__reduce_add_sync(0xffffffffu, n) >= (uint32_t)c) T = t;
  }
  if (lane == 0) p.thr[rr * p.state_ld] = T;
}

constexpr int CS_T = 256;       // threads of a select block
constexpr int CS_SMALL = 256;   // keys of the boundary bin resolved one per thread

// Step 4: one block per row.  Dynamic shared memory: the row's candidate keys (cap) and a
// bitmap of the selected positions (ceil(vis / 32) words, sized for the launch's longest
// row).  With d = key - bound over the candidates: 2048-bin histograms of 11-bit digits of
// d, from the top of its range, locate the bin of the k-th largest key (one level when
// that bin holds at most CS_SMALL keys, which is the usual case; up to three otherwise);
// candidates above that bin are selected outright, and those in it go to a small list in
// which each thread ranks one key against the others by (key descending, position
// ascending), the ranks below k - (count above) being selected.  A block scan over the
// bitmap writes the positions in ascending order.  A row with more than CS_SMALL keys
// equal to the k-th (massive ties) is marked -2 for the exact path.
__global__ void __launch_bounds__(CS_T) topk_cand_select_kernel(const FusedTopkParams p, int words) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem_raw);
  uint32_t* selw = ckey + p.cap;
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t total, bin, above, dmax, nsmall;
  __shared__ uint32_t skey[CS_SMALL];
  __shared__ int spos[CS_SMALL];
  const long long rr = blockIdx.x;
  int vis, kg;
  fused_row_geometry(p, p.row_begin + rr, vis, kg);
  const int k = p.k;
  int* out = p.indices + rr * k;
  if (vis <= k) {
    for (int j = threadIdx.x; j < k; j += CS_T) out[j] = j < vis ? j : -1;
    return;
  }
  // the row's bound and count sit in its own output slots: read them before any write
  const uint32_t n = p.cnt[rr * p.state_ld];
  const uint32_t T = p.thr[rr * p.state_ld];
  if (n < (uint32_t)k || n > (uint32_t)p.cap) {  // block-uniform
    if (threadIdx.x == 0) {
      out[0] = -2;
      atomicExch(p.flag, 1);
    }
    return;
  }
  const uint2* src = p.cand + rr * p.cap;
  uint32_t dm = 0;
  // four independent loads in flight per thread
  for (uint32_t j0 = threadIdx.x; j0 < n; j0 += 4 * CS_T) {
    uint32_t kk[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = j0 + u * CS_T;
      kk[u] = j < n ? __ldg(&src[j].x) : T;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = j0 + u * CS_T;
      if (j < n) ckey[j] = kk[u];
      dm = max(dm, kk[u] - T);
    }
  }
  dm = __reduce_max_sync(0xffffffffu, dm);
  const int W = (vis + 31) / 32;
  for (int j = threadIdx.x; j < W; j += CS_T) selw[j] = 0u;
  if (threadIdx.x == 0) {
    dmax = 0;
    nsmall = 0;
  }
  __syncthreads();
  if ((threadIdx.x & 31) == 0) atomicMax(&dmax, dm);
  __syncthreads();
  // radix levels over d = key - bound (11 bits each, from the top of the range): each level
  // narrows to the bin holding the rem-th largest of the keys that share the prefix so far,
  // and stops once that bin is small (or the last bits are reached)
  const int nbits = 32 - __clz((int)dmax);
  int shift = max(0, nbits - 11);
  uint32_t prefix = 0, pmask = 0, rem = (uint32_t)k, in_bin = 0;
#pragma unroll 1
  while (true) {
    for (int j = threadIdx.x; j < 2048; j += CS_T) hist[j] = 0u;
    __syncthreads();
    for (uint32_t j = threadIdx.x; j < n; j += CS_T) {
      const uint32_t d = ckey[j] - T;
      if ((d & pmask) == prefix) atomicAdd(&hist[(d >> shift) & 2047u], 1u);
    }
    __syncthreads();
    find_bin<CS_T, 2048>(hist, rem, warp_sums, &total, &bin, &above);
    in_bin = hist[bin];
    prefix |= bin << shift;
    pmask |= 2047u << shift;
    rem -= above;
    if (in_bin <= (uint32_t)CS_SMALL || shift == 0) break;
    shift = max(0, shift - 11);
    __syncthreads();  // every thread has read hist[bin] before the next level clears it
  }
  if (in_bin > (uint32_t)CS_SMALL) {  // block-uniform: more than CS_SMALL equal keys
    if (threadIdx.x == 0) {
      out[0] = -2;
      atomicExch(p.flag, 1);
    }
    return;
  }
  for (uint32_t j0 = threadIdx.x; j0 < n; j0 += 4 * CS_T) {
    uint32_t md[4];
    int sp[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t j = j0 + u * CS_T;
      md[u] = j < n ? (ckey[j] - T) & pmask : 0u;
      sp[u] = (j < n && md[u] >= prefix) ? (int)__ldg(&src[j].y) : -1;  // (L2 hits: just read)
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (sp[u] < 0) continue;
      const int s = sp[u];
      if (md[u] > prefix) {
        atomicOr(&selw[s >> 5], 1u << (s & 31));
      } else {
        const uint32_t slot = atomicAdd(&nsmall, 1u);
        skey[slot] = ckey[j0 + u * CS_T];
        spos[slot] = s;
      }
    }
  }
  __syncthreads();
  const uint32_t m = nsmall;  // == in_bin <= CS_SMALL
  if (threadIdx.x < m) {
    const uint32_t key = skey[threadIdx.x];
    const int s = spos[threadIdx.x];
    uint32_t rank = 0;
    for (uint32_t f = 0; f < m; ++f) rank += skey[f] > key || (skey[f] == key && spos[f] < s);
    if (rank < rem) atomicOr(&selw[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  // a contiguous run of words per thread, so that a block scan gives position order
  const int wpt = (W + CS_T - 1) / CS_T;
  const int w0 = min(W, (int)threadIdx.x * wpt), w1 = min(W, w0 + wpt);
  uint32_t mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(selw[w]);
  uint32_t o = block_excl_scan<CS_T>(mine, warp_sums, &total);  // the block selects exactly k
  for (int w = w0; w < w1; ++w) {
    uint32_t x = selw[w];
    while (x) {
      if (o < (uint32_t)k) out[o] = w * 32 + (__ffs(x) - 1);
      ++o;
      x &= x - 1u;
    }
  }
}

}  // namespace dsa

namespace dsa_host {

// (Indexer2Pass, indexer2_shape and indexer2_pass_launch come from indexer2.cu, earlier in
// this unity build.)
static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// The fused path's sampling stride, sampled-row pitch and candidates per row for score
// rows of `ld` positions, or ok = false where it does not apply (other indexer shapes, rows
// past 524288 positions, k < 4 (a row's bound and count borrow two of its k output slots),
// or a chunk scratch too small for 2k candidates per row).
struct FusedPlan {
  bool ok = false;
  int S = 1;
  long long ld_s = 0;
  int cap = 0;
};

static FusedPlan fused_plan(long long ld, int k, int H_I, int d_I) {
  FusedPlan f;
  if (!indexer2_shape(H_I, d_I) || ld > 524288 || k > 4096 || k < 4) return f;
  f.S = 4;
  while (f.S < 1024 && (ld + f.S - 1) / f.S > 1024) f.S *= 2;
  f.ld_s = ((ld + f.S - 1) / f.S + 1 + 3) / 4 * 4;
  // the candidate lists share each row's ld * 4 bytes of the score scratch with the repair
  // pass, which writes full score rows over them
  f.cap = (int)std::min<long long>(8192, (ld * 4 - 64) / 8) / 4 * 4;
  f.ok = f.cap >= 2 * k && (ld + f.S - 1) / f.S + 1 <= 32 * dsa::SB_KPL;
  return f;
}

static long long score_ld(int max_seqlen_k) { return ((long long)std::max(max_seqlen_k, 1) + 3) / 4 * 4; }

// Scratch of index_topk_launch: the fp32 score rows of one chunk (also holding the fused
// path's sampled rows and candidate lists) and the repair flag after them.
size_t index_topk_workspace_bytes(long long chunk_rows, int max_seqlen_k) {
  return up256((size_t)chunk_rows * (size_t)score_ld(max_seqlen_k) * 4) + 256;
}

int indexer_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                   long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k, int H_I, int d_I,
                   long long row_begin, long long row_end, float* scores, long long ld, cudaStream_t stream);
int topk_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch, long long row_begin,
                long long row_end, int k, int* indices, int max_vis, void* ws, size_t ws_bytes, cudaStream_t stream);
int topk_marked_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                       long long row_begin, long long row_end, int k, int* indices, int* flag_reset,
                       cudaStream_t stream);

// Selected sets of the query rows [row_begin, row_end) (indices points at row row_begin's
// slots): the fused path or the separate indexer and top-k passes per chunk, as `fused`
// asks (0 separate, 1 automatic, 2 fused where fused_plan allows it).
int index_topk_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                      int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k, int H_I,
                      int d_I, int k, long long row_begin, long long row_end, long long chunk_rows, int* indices,
                      void* ws, int fused, cudaStream_t stream) {
  const long long ld = score_ld(max_seqlen_k);
  const FusedPlan plan = fused_plan(ld, k, H_I, d_I);
  const size_t region = (size_t)chunk_rows * (size_t)ld * 4;  // the chunk's score rows
  float* scores = static_cast<float*>(ws);
  int* flag = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + up256(region));
  // Rows [fused_begin, row_end) take the fused path.  It pays where rows see many more
  // positions than a row keeps candidates (a row of at most `cap` visible positions keeps
  // them all, as 8-byte pairs, so it is cheaper on the separate passes): not at all for
  // score rows shorter than 65536 (measured: slower at 16K and 32K, faster at 128K), and for
  // one self-attention sequence (batch 1, Lq == Lk, row r sees r + 1 positions) not in the
  // leading chunks whose rows see at most 2 cap positions.
  // (fused: 0 = separate passes, 1 = that choice, 2 = the fused path wherever the plan allows)
  long long fused_begin = row_end;
  if (plan.ok && fused == 2) {
    fused_begin = row_begin;
  } else if (plan.ok && fused == 1 && ld >= 65536) {
    fused_begin = row_begin;
    if (batch == 1 && total_q == total_k)
      while (fused_begin < row_end && std::min(row_end, fused_begin + chunk_rows) <= 2LL * plan.cap)
        fused_begin += chunk_rows;
  }
  if (fused_begin > row_begin) {
    for (long long r0 = row_begin; r0 < fused_begin; r0 += chunk_rows) {
      const long long r1 = std::min(fused_begin, r0 + chunk_rows);
      int st = indexer_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_q, max_seqlen_k, H_I,
                              d_I, r0, r1, scores, ld, stream);
      if (st != DSA_OK) return st;
      st = topk_launch(scores, ld, cu_q, cu_k, batch, r0, r1, k, indices + (r0 - row_begin) * k,
                       (int)std::min<long long>(ld, 0x7FFFFFFF), nullptr, 0, stream);
      if (st != DSA_OK) return st;
    }
    if (fused_begin == row_end) return DSA_OK;
  }
  static DeviceFlag attr_done;
  // at most 8192 candidate keys and a bitmap of 524288 bits: 96 KiB
  const int words = (int)((ld + 31) / 32);
  const int select_smem = plan.cap * 4 + words * 4;
  if (!attr_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_cand_select_kernel,
                                                cudaFuncAttributeMaxDynamicSharedMemorySize, 96 * 1024);
    if (e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  dsa::FusedTopkParams fp;
  fp.S = plan.S;
  fp.ld_s = plan.ld_s;
  fp.cu_q = cu_q;
  fp.cu_k = cu_k;
  fp.batch = batch;
  fp.k = k;
  fp.cap = plan.cap;
  fp.state_ld = k;
  fp.flag = flag;
  // A. sampled scores and bounds of every row, in groups whose sampled rows fit the scratch
  const long long group = std::max<long long>(1, (long long)(region / ((size_t)plan.ld_s * 4)));
  for (long long g0 = fused_begin; g0 < row_end; g0 += group) {
    const long long g1 = std::min(row_end, g0 + group);
    Indexer2Pass ps;
    ps.key_stride = plan.S;
    float* samples = scores;
    int st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, g0,
                                  g1, samples, plan.ld_s, false, ps, stream);
    if (st != DSA_OK) return st;
    fp.samples = samples;
    fp.row_begin = g0;
    fp.rows = g1 - g0;
    fp.thr = reinterpret_cast<uint32_t*>(indices + (g0 - row_begin) * k + (k - 1));
    fp.cnt = reinterpret_cast<uint32_t*>(indices + (g0 - row_begin) * k + (k - 2));
    dsa::topk_sample_bound_kernel<<<(unsigned)((fp.rows + dsa::SB_WARPS - 1) / dsa::SB_WARPS), dsa::SB_WARPS * 32, 0,
                                    stream>>>(fp);
    if ((st = last_launch_status()) != DSA_OK) return st;
  }
  if (cudaError_t e_ = cudaMemsetAsync(flag, 0, sizeof(int), stream); e_ != cudaSuccess) return cuda_fail(e_);
  // B. per chunk: candidates, selection, repair of the rows the bound failed for
  uint2* cand = reinterpret_cast<uint2*>(ws);
  for (long long r0 = fused_begin; r0 < row_end; r0 += chunk_rows) {
    const long long r1 = std::min(row_end, r0 + chunk_rows);
    int* out = indices + (r0 - row_begin) * k;
    fp.row_begin = r0;
    fp.rows = r1 - r0;
    fp.thr = reinterpret_cast<uint32_t*>(out + (k - 1));
    fp.cnt = reinterpret_cast<uint32_t*>(out + (k - 2));
    fp.cand = cand;
    fp.indices = out;
    Indexer2Pass pf;
    pf.thr = fp.thr;
    pf.cnt = fp.cnt;
    pf.state_ld = k;
    pf.cand = cand;
    pf.cap = plan.cap;
    int st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, r0,
                                  r1, nullptr, ld, true, pf, stream);
    if (st != DSA_OK) return st;
    dsa::topk_cand_select_kernel<<<(unsigned)fp.rows, dsa::CS_T, select_smem, stream>>>(fp, words);
    if ((st = last_launch_status()) != DSA_OK) return st;
    // both launches do nothing unless a row of the chunk raised the flag (the second clears it)
    Indexer2Pass pr;
    pr.mark = out;
    pr.mark_ld = k;
    pr.run_flag = flag;
    st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, r0, r1,
                              scores, ld, false, pr, stream);
    if (st != DSA_OK) return st;
    st = topk_marked_launch(scores, ld, cu_q, cu_k, batch, r0, r1, k, out, flag, stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

}  // namespace dsa_host
