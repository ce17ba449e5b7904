// Fused lightning indexer -> deterministic top-k (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1 (the indexer scans
// every visible position and each token keeps its 2048 best) and section 8 (the top-k
// must be deterministic).  The separate path writes every score of a row chunk to an fp32
// scratch and reads it back to select (34 GB each way at 128K context); here the indexer
// keeps only the scores that can still be among a row's k largest.
//
// Per row chunk:
//   1. sampled scores: the CTA-pair indexer over every S-th indexer key (S chosen so that
//      a full row has about 1024 samples), about 1/S of the indexer's work;
//   2. bound: per row, the c-th largest sampled score, c = m + 3 sqrt(m) + 8 with m = k / S
//      (the number of samples expected at or above the row's k-th largest score), cut to
//      22 key bits.  Rows with at most `cap` visible positions get no bound (all pass);
//   3. fused indexer: every score whose order key reaches the row's bound is appended to
//      the row's candidate list as (key, position); no score matrix is written;
//   4. select: per row, the exact k-th largest key K* over the candidates by radix levels
//      over (key - bound), then the selected positions through two bitmaps over the row
//      (keys > K*, ties at K*; the lowest-positioned `remaining` ties are kept) and a
//      block scan, so the output is ascending whatever order the candidates arrived in.
//      A row with fewer than k candidates (an unlucky sample) or more than `cap` (huge
//      ties) is marked -2 and raises the chunk's repair flag;
//   5. repair: only if the flag is raised, the indexer writes the full score rows of the
//      marked rows' blocks to the scratch and the exact top-k selects them.
// Every candidate list holds exactly the positions whose key reaches the bound, and the
// bound only decides how many positions are kept, never which of them are selected: the
// result is the exact top-k of the rows' scores, bit for bit the one the separate path
// returns on the same scores.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct FusedTopkParams {
  const float* samples;  // [rows, ld_s] sampled scores of the chunk
  long long ld_s;
  int S;                 // key stride of the samples
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin;   // first row of the chunk
  int k;
  int cap;               // candidates kept per row
  uint32_t* thr;         // [rows] bound (order key) per row
  uint32_t* cnt;         // [rows] candidates appended per row
  int* flag;             // set when a row needs the repair pass
  const uint2* cand;     // [rows, cap] (order key, position)
  int* indices;          // [rows, k] output of the chunk's rows
  int words;             // bitmap words per row: ceil(longest visible range / 32)
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

constexpr int SB_T = 256;   // threads of a bound block
constexpr int SB_PER = 32;  // sampled scores per thread: rows of up to 8192 samples

// Step 2: one block per row of the chunk.  Also clears the row's candidate count and
// (block 0) the chunk's repair flag.
__global__ void __launch_bounds__(SB_T) topk_sample_bound_kernel(const FusedTopkParams p) {
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t total, bin, above;
  const long long rr = blockIdx.x;
  if (rr == 0 && threadIdx.x == 0) *p.flag = 0;
  if (threadIdx.x == 0) p.cnt[rr] = 0;
  int vis, kg;
  fused_row_geometry(p, p.row_begin + rr, vis, kg);
  const long long S = p.S;
  const int k0s = (int)((kg + S - 1) / S);
  const int ns = (int)((kg + (long long)vis + S - 1) / S) - k0s;  // sampled positions of the row
  const float m = (float)p.k / (float)S;
  const int c = (int)ceilf(m + 3.f * sqrtf(m) + 8.f);
  if (vis <= p.cap || c >= ns) {  // block-uniform: every visible position is a candidate
    if (threadIdx.x == 0) p.thr[rr] = 0u;
    return;
  }
  const float* src = p.samples + rr * p.ld_s;
  uint32_t sk[SB_PER];
#pragma unroll
  for (int u = 0; u < SB_PER; ++u) {
    const int j = u * SB_T + threadIdx.x;
    sk[u] = j < ns ? float_order_key(__ldg(src + j)) : 0u;
  }
  // the c-th largest sampled key to 22 bits, by two radix levels (11 + 11 key bits)
  uint32_t sp = 0, sm = 0, rem = (uint32_t)c;
#pragma unroll 1
  for (int lv = 0; lv < 2; ++lv) {
    const int shift = lv == 0 ? 21 : 10;
    for (int j = threadIdx.x; j < 2048; j += SB_T) hist[j] = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < SB_PER; ++u) {
      const int j = u * SB_T + threadIdx.x;
      // one counter update per distinct bin and warp: a row's samples share their top bits
      const bool act = j < ns && (sk[u] & sm) == sp;
      const uint32_t b = act ? (sk[u] >> shift) & 2047u : 0xFFFFFFFFu;
      const uint32_t peers = __match_any_sync(0xffffffffu, b);
      if (act && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[b], (uint32_t)__popc(peers));
    }
    __syncthreads();
    find_bin<SB_T, 2048>(hist, rem, warp_sums, &total, &bin, &above);
    sp |= bin << shift;
    sm |= 2047u << shift;
    rem -= above;
  }
  if (threadIdx.x == 0) p.thr[rr] = sp;
}

constexpr int CS_T = 512;  // threads of a select block

// Step 4: one block per row of the chunk.  Dynamic shared memory: the row's candidates
// (cap keys, cap positions) and two bitmaps of `words` words.
__global__ void __launch_bounds__(CS_T) topk_cand_select_kernel(const FusedTopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* ckey = reinterpret_cast<uint32_t*>(smem_raw);
  int* cpos = reinterpret_cast<int*>(ckey + p.cap);
  uint32_t* selw = reinterpret_cast<uint32_t*>(cpos + p.cap);  // keys > K*, then the selection
  uint32_t* tiew = selw + p.words;                              // keys == K*
  __shared__ uint32_t hist[2048];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t total, bin, above, dmax;
  const long long rr = blockIdx.x;
  int vis, kg;
  fused_row_geometry(p, p.row_begin + rr, vis, kg);
  const int k = p.k;
  int* out = p.indices + rr * k;
  if (vis <= k) {
    for (int j = threadIdx.x; j < k; j += CS_T) out[j] = j < vis ? j : -1;
    return;
  }
  const uint32_t n = p.cnt[rr];
  if (n < (uint32_t)k || n > (uint32_t)p.cap) {  // block-uniform
    if (threadIdx.x == 0) {
      out[0] = -2;
      atomicExch(p.flag, 1);
    }
    return;
  }
  const uint2* src = p.cand + rr * p.cap;
  for (uint32_t j = threadIdx.x; j < n; j += CS_T) {
    const uint2 e = src[j];
    ckey[j] = e.x;
    cpos[j] = (int)e.y;
  }
  const int W = (vis + 31) / 32;
  for (int j = threadIdx.x; j < W; j += CS_T) {
    selw[j] = 0u;
    tiew[j] = 0u;
  }
  __syncthreads();
  uint32_t kstar, remaining;
  select_relative<CS_T>(ckey, (int)n, p.thr[rr], (uint32_t)k, hist, warp_sums, &total, &bin, &above, &dmax, kstar,
                        remaining);
  for (uint32_t j = threadIdx.x; j < n; j += CS_T) {
    const uint32_t key = ckey[j];
    const int s = cpos[j];
    if (key > kstar) atomicOr(&selw[s >> 5], 1u << (s & 31));
    else if (key == kstar) atomicOr(&tiew[s >> 5], 1u << (s & 31));
  }
  __syncthreads();
  // a contiguous run of words per thread, so that block scans give position order
  const int wpt = (W + CS_T - 1) / CS_T;
  const int w0 = min(W, (int)threadIdx.x * wpt), w1 = min(W, w0 + wpt);
  uint32_t ties = 0;
  for (int w = w0; w < w1; ++w) ties += __popc(tiew[w]);
  uint32_t before = block_excl_scan<CS_T>(ties, warp_sums, &total);
  uint32_t mine = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t x = tiew[w];
    const uint32_t c = __popc(x);
    if (before >= remaining) {
      x = 0u;
    } else if (before + c > remaining) {  // keep the lowest (remaining - before) tie positions
      uint32_t keep = 0u;
      for (uint32_t t = before; t < remaining; ++t) {
        const uint32_t low = x & (~x + 1u);
        keep |= low;
        x ^= low;
      }
      x = keep;
    }
    before += c;
    const uint32_t sel = selw[w] | x;
    selw[w] = sel;
    mine += __popc(sel);
  }
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
int topk_marked_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch,
                       long long row_begin, long long row_end, int k, int* indices, cudaStream_t stream);

static size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// The fused path's sampling stride, sampled-row pitch and candidates per row for score
// rows of `ld` positions, or ok = false where it does not apply (other indexer shapes, rows
// past 512K positions, or a chunk scratch too small for 2k candidates per row).
struct FusedPlan {
  bool ok = false;
  int S = 1;
  long long ld_s = 0;
  int cap = 0;
};

static FusedPlan fused_plan(long long ld, int k, int H_I, int d_I) {
  FusedPlan f;
  if (!indexer2_shape(H_I, d_I) || ld > 524288 || k > 4096) return f;
  f.S = 4;
  while (f.S < 128 && (ld + f.S - 1) / f.S > 1024) f.S *= 2;
  f.ld_s = ((ld + f.S - 1) / f.S + 1 + 3) / 4 * 4;
  // the candidate lists, the sampled rows and the per-row bound and count share each row's
  // ld * 4 bytes of the score scratch (the repair pass writes the full rows over them)
  const long long per_row = ld * 4 - f.ld_s * 4 - 8 - 64;
  f.cap = (int)std::min<long long>(8192, per_row / 8) / 4 * 4;
  f.ok = f.cap >= 2 * k && (ld + f.S - 1) / f.S + 1 <= dsa::SB_T * dsa::SB_PER;
  return f;
}

static long long score_ld(int max_seqlen_k) { return ((long long)std::max(max_seqlen_k, 1) + 3) / 4 * 4; }

// Scratch of index_topk_launch: the fp32 score rows of one chunk (also holding the fused
// path's candidates, samples, bounds and counts) and the repair flag after them.
size_t index_topk_workspace_bytes(long long chunk_rows, int max_seqlen_k) {
  return up256((size_t)chunk_rows * (size_t)score_ld(max_seqlen_k) * 4) + 256;
}

int indexer_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                   long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k, int H_I, int d_I,
                   long long row_begin, long long row_end, float* scores, long long ld, cudaStream_t stream);
int topk_launch(const float* scores, long long ld, const int* cu_q, const int* cu_k, int batch, long long row_begin,
                long long row_end, int k, int* indices, int max_vis, void* ws, size_t ws_bytes, cudaStream_t stream);

// Selected sets of every query row, chunk by chunk: the fused path where fused_plan allows
// it (or `fused` is 1), the separate indexer and top-k passes otherwise (or `fused` is 0).
int index_topk_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                      int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k, int H_I,
                      int d_I, int k, long long chunk_rows, int* indices, void* ws, int fused, cudaStream_t stream) {
  const long long ld = score_ld(max_seqlen_k);
  const FusedPlan plan = fused_plan(ld, k, H_I, d_I);
  const bool use_fused = plan.ok && fused != 0;
  float* scores = static_cast<float*>(ws);
  int* flag = reinterpret_cast<int*>(static_cast<uint8_t*>(ws) + up256((size_t)chunk_rows * (size_t)ld * 4));
  static DeviceFlag attr_done;
  int select_smem = 0;
  if (use_fused) {
    // at most 8192 candidates and two bitmaps of 524288 bits: 192 KiB
    select_smem = plan.cap * 8 + 2 * (int)((ld + 31) / 32) * 4;
    if (!attr_done) {
      const cudaError_t e_ = cudaFuncSetAttribute(dsa::topk_cand_select_kernel,
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, 192 * 1024);
      if (e_ != cudaSuccess) return cuda_fail(e_);
      attr_done = true;
    }
  }
  for (long long r0 = 0; r0 < total_q; r0 += chunk_rows) {
    const long long r1 = std::min(total_q, r0 + chunk_rows);
    const long long rows = r1 - r0;
    int* out = indices + r0 * k;
    // the fused path's lists, samples, bounds and counts must fit the chunk's score rows
    const size_t fused_bytes = up256((size_t)rows * plan.cap * 8) + up256((size_t)rows * plan.ld_s * 4) +
                               2 * up256((size_t)rows * 4);
    if (!use_fused || fused_bytes > (size_t)rows * (size_t)ld * 4) {
      int st = indexer_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_q, max_seqlen_k, H_I,
                              d_I, r0, r1, scores, ld, stream);
      if (st != DSA_OK) return st;
      st = topk_launch(scores, ld, cu_q, cu_k, batch, r0, r1, k, out, (int)std::min<long long>(ld, 0x7FFFFFFF),
                       nullptr, 0, stream);
      if (st != DSA_OK) return st;
      continue;
    }
    uint8_t* wp = static_cast<uint8_t*>(ws);
    uint2* cand = reinterpret_cast<uint2*>(wp);
    wp += up256((size_t)rows * plan.cap * 8);
    float* samples = reinterpret_cast<float*>(wp);
    wp += up256((size_t)rows * plan.ld_s * 4);
    uint32_t* thr = reinterpret_cast<uint32_t*>(wp);
    wp += up256((size_t)rows * 4);
    uint32_t* cnt = reinterpret_cast<uint32_t*>(wp);
    dsa::FusedTopkParams fp;
    fp.samples = samples;
    fp.ld_s = plan.ld_s;
    fp.S = plan.S;
    fp.cu_q = cu_q;
    fp.cu_k = cu_k;
    fp.batch = batch;
    fp.row_begin = r0;
    fp.k = k;
    fp.cap = plan.cap;
    fp.thr = thr;
    fp.cnt = cnt;
    fp.flag = flag;
    fp.cand = cand;
    fp.indices = out;
    fp.words = (int)((ld + 31) / 32);
    // 1. sampled scores
    Indexer2Pass ps;
    ps.key_stride = plan.S;
    int st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, r0,
                                  r1, samples, plan.ld_s, false, ps, stream);
    if (st != DSA_OK) return st;
    // 2. per-row bound (and zeroed counts, cleared repair flag)
    dsa::topk_sample_bound_kernel<<<(unsigned)rows, dsa::SB_T, 0, stream>>>(fp);
    if ((st = last_launch_status()) != DSA_OK) return st;
    // 3. fused indexer: candidates instead of scores
    Indexer2Pass pf;
    pf.thr = thr;
    pf.cnt = cnt;
    pf.cand = cand;
    pf.cap = plan.cap;
    st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, r0, r1,
                              nullptr, ld, true, pf, stream);
    if (st != DSA_OK) return st;
    // 4. exact selection over the candidates
    dsa::topk_cand_select_kernel<<<(unsigned)rows, dsa::CS_T, select_smem, stream>>>(fp);
    if ((st = last_launch_status()) != DSA_OK) return st;
    // 5. repair of marked rows (both launches do nothing unless the flag is raised)
    Indexer2Pass pr;
    pr.mark = out;
    pr.mark_ld = k;
    pr.run_flag = flag;
    st = indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, r0, r1,
                              scores, ld, false, pr, stream);
    if (st != DSA_OK) return st;
    st = topk_marked_launch(scores, ld, cu_q, cu_k, batch, r0, r1, k, out, stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

}  // namespace dsa_host
