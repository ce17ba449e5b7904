// Sparse GQA attention over the top-k selected positions on the tensor cores (sm_100a,
// prefill, d = 128, 8 query heads per KV head): the entry point dsa_sparse_attn_prefill_tc.
// The default entry (sparse_attn_kernel, warp-level MMA) is the faster of the two on B200:
// the selected rows arrive from L2 at a latency of microseconds under this load, so the
// gather needs about 200 KB in flight per SM; that kernel's per-warp rings keep nearly all
// of their 224 KB in flight, while here each 32 KB stage is also held through S, the
// softmax and P.V (measured at 128K: 89.5 against 39.1 ms).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: attention runs only
// over the positions the indexer selected, and DSA is adapted to GQA with one selected set
// per token, shared by the query heads of its KV group.  Same operation, validity rule and
// results as sparse_attn_kernel (sparse_attn.cu): a slot s of row t counts when
// 0 <= s < vis(t); lse is the natural-log normaliser; O is divided by the sum of the
// bf16-rounded weights that enter the P.V product.
//
// Work item: one (query row t, KV head g); the KV head is the slowest index, so the CTAs in
// flight gather from one head's K/V rows (64 MiB at 128K context), which stay in L2.  A tile
// is 128 consecutive slots of the row's selection, in swap-AB form so that the selected
// keys fill the MMA's M = 128:
//   S^T [128 slots x 16]  = K_tile [128 x d] . Q_g^T [d x 16]        (columns 0-7: the heads)
//   O^T [d x 16]         += V_tile^T [d x 128 slots] . P^T [128 x 16]
// N = 16 is the smallest N of the M = 128 shape; columns 8-15 are never read.  Roles of the
// 16 warps of a persistent CTA (one per SM, 226 KB of shared memory):
//   warp 0        the item's slot list (one bulk copy into shared memory, read there by
//                 the copy and epilogue warps) and Q_g (8 rows of 256 B, cp.async), 2 stages;
//   warp 1        TMEM owner and MMA issuer (S of tile n + 1 is issued before P.V of tile n);
//   warps 4-7     epilogue: thread i owns slot i of S^T (TMEM lane i) and dimension i of O^T;
//   warps 2-3, 8-10  copy K rows, warps 11-15 V rows, 16-byte cp.async into 3-stage rings in
//                 the 128-byte-swizzled layout (zero-filled for invalid slots; eight lanes
//                 per row), completion signalled with cp.async.mbarrier.arrive.noinc.
// Online softmax in the log2 domain: the running max of a head moves only when a tile
// exceeds it by more than 8, decided for all 128 epilogue threads at once by one barrier
// reduction per tile; in that case the tile's maxima are reduced through shared memory and
// O^T is rescaled in tensor memory (after the previous P.V completed).  Every wait is
// bounded (detail codes 138-153).
#include "common.cuh"

namespace dsa {

struct SGParams {
  const uint16_t* Q;    // [rows, Hq, 128]
  const uint16_t* K;    // [total_k, Hkv, 128]
  const uint16_t* V;
  const int* indices;   // [rows, k] (16-byte aligned, k a multiple of 16, at most 2048)
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long rows;
  int Hq, Hkv, k;
  float scale_log2;
  uint16_t* O;          // [rows, Hq, 128]
  float* lse;           // [rows, Hq] or null
  const uint8_t* skip_rows;  // optional [rows]: rows another kernel computes
};

struct SGCfg {
  static constexpr int TILE_BYTES = 128 * 128 * 2;  // 128 rows x 256 B (two 64-element panels)
  static constexpr int PANEL = 128 * 128;
  static constexpr int KS = 3, VS = 3;
  static constexpr int SMALL = 16 * 128 * 2;        // a 16 x 128 bf16 operand (Q or P^T)
  static constexpr int SMALL_PANEL = 16 * 128;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KS * TILE_BYTES;
  static constexpr int OFF_Q = OFF_V + VS * TILE_BYTES;
  static constexpr int OFF_P = OFF_Q + 2 * SMALL;
  static constexpr int MAX_K = 2048;                  // selection slots per row
  static constexpr int OFF_IDX = OFF_P + 2 * SMALL;  // 2 x the item's slot list (int32)
  // [4][8] tile maxima, [4][16] item sums, [8] per-warp wait outcomes
  static constexpr int OFF_RED = OFF_IDX + 2 * MAX_K * 4;
  static constexpr int OFF_BAR = OFF_RED + 4 * 8 * 4 + 4 * 16 * 4 + 8 * 4;
  // q_full[2] q_empty[2] k_full[KS] k_empty[KS] v_full[VS] v_empty[VS] s_full[2] s_empty[2]
  // p_full[2] p_empty[2] o_full[2] o_empty[2] mma_done idx_full[2] idx_empty[2]
  static constexpr int NUM_BARS = 4 + 2 * KS + 2 * VS + 8 + 4 + 1 + 4;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 512;
  static constexpr int GK = 5, GV = 5;  // copy warps for K and for V
  static constexpr int TMEM_COLS = 64;  // S^T buffers at 0, 16; O^T buffers at 32, 48
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 16);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 16) | kIdescAMnMajor;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "swizzle atoms need 1024-byte alignment");
};

// The (row, KV head) of a work item, its sequence's first key row and the row's visible
// keys; false for rows another kernel computes.
struct SGItem {
  long long row;
  int g, kbase, vis;
};
__device__ __forceinline__ bool sg_item(const SGParams& p, long long item, SGItem& it) {
  it.g = (int)(item / p.rows);
  it.row = item - (long long)it.g * p.rows;
  if (p.skip_rows && p.skip_rows[it.row]) return false;
  int lo = 0, hi = p.batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)p.cu_q[mid] <= it.row) lo = mid; else hi = mid;
  }
  it.kbase = p.cu_k[lo];
  it.vis = causal_vis((int)(it.row - p.cu_q[lo]), p.cu_q[lo + 1] - p.cu_q[lo], p.cu_k[lo + 1] - it.kbase);
  return true;
}

// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global memory
// into shared memory, completing as transaction bytes on `bar`.
__device__ __forceinline__ void sg_bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Copies the K (or V) rows of one tile's 128 slots (`nslots` of them inside the selection)
// into `dst` (two 16 KB panels, 128-byte swizzle), zero-filling invalid slots.  Eight lanes
// per row: each warp instruction moves whole 128-byte halves of four rows (as coalesced as
// two full rows per instruction), and the row's slot and address are worked out once for its
// two halves.  This warp takes the groups of four rows wg, wg + nw, ...  Arrives on `bar`
// once its copies have landed.
__device__ __forceinline__ void sg_copy_tile(uint32_t dst, const uint16_t* base, const int* slots, int nslots,
                                             int kbase, int vis, long long row_stride, int nw, int wg, int lane,
                                             uint64_t* bar) {
  const int sub = lane >> 3, c = lane & 7;
#pragma unroll 2
  for (int q = wg; q < 32; q += nw) {
    const int r = 4 * q + sub;
    const int s = r < nslots ? slots[r] : -1;
    const bool valid = (unsigned)s < (unsigned)vis;
    const uint16_t* src = base + (valid ? (long long)(kbase + s) * row_stride : 0LL) + c * 8;
    const uint32_t d0 = dst + r * 128 + ((c ^ (r & 7)) * 16);
    cp_async_16(d0, src, valid);                       // dims 8c .. 8c + 7 (panel 0)
    cp_async_16(d0 + SGCfg::PANEL, src + 64, valid);   // dims 64 + 8c .. (panel 1)
  }
  cp_async_mbar_arrive(bar);
}

__global__ void __launch_bounds__(SGCfg::THREADS, 1) sa_gather_tc_kernel(const SGParams p) {
  using C = SGCfg;
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 2;
  uint64_t* k_full = bars + 4;
  uint64_t* k_empty = k_full + C::KS;
  uint64_t* v_full = k_empty + C::KS;
  uint64_t* v_empty = v_full + C::VS;
  uint64_t* s_full = v_empty + C::VS;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_full + 4;
  uint64_t* p_empty = s_full + 6;
  uint64_t* o_full = s_full + 8;
  uint64_t* o_empty = s_full + 10;
  uint64_t* mma_done = s_full + 12;
  uint64_t* idx_full = s_full + 13;
  uint64_t* idx_empty = s_full + 15;
  const int* idx_s = reinterpret_cast<const int*>(smem + C::OFF_IDX);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  float* red_max = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* red_sum = red_max + 4 * 8;
  volatile int* red_ok = reinterpret_cast<volatile int*>(red_sum + 4 * 16);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 32);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&p_empty[i], 1);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_empty[i], 4);
      mbar_init(&idx_full[i], 1);
      mbar_init(&idx_empty[i], C::GK + C::GV + 4);  // one arrival per copy and epilogue warp
    }
    for (int i = 0; i < C::KS; ++i) {
      mbar_init(&k_full[i], C::GK * 32);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::VS; ++i) {
      mbar_init(&v_full[i], C::GV * 32);
      mbar_init(&v_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  // rows 8-15 of the Q and P^T operands are never written by the pipeline: zero them once
  // (they only feed columns 8-15 of S^T and O^T, which nothing reads)
  for (int e = threadIdx.x; e < 4 * 2 * 8 * 128 / 16; e += C::THREADS) {
    const int buf = e / 128, rem = e % 128;  // 4 operands x 2 panels x rows 8-15 x 8 chunks
    const int pn = rem / 64, r = 8 + (rem % 64) / 8, ch = rem % 8;
    *reinterpret_cast<uint4*>(smem + C::OFF_Q + buf * C::SMALL + pn * C::SMALL_PANEL + r * 128 + ch * 16) =
        make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_shared();
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const long long n_items = p.rows * p.Hkv;
  const int T = (p.k + 127) / 128;  // tiles per item
  const long long kv_stride = (long long)p.Hkv * 128;

  if (warp == 0) {
    // ------------------------------------------------------------ each item's slot list (one
    // bulk copy, read from shared memory by the copy and epilogue warps) and Q_g
    long long m = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      SGItem it;
      if (!sg_item(p, item, it)) continue;
      const int qs = (int)(m & 1);
      if (lane == 0) {
        ok = mbar_wait(&idx_empty[qs], (uint32_t)((m >> 1) & 1) ^ 1u, abort_flag, 151) &&
             mbar_wait(&q_empty[qs], (uint32_t)((m >> 1) & 1) ^ 1u, abort_flag, 140);
        if (ok) {
          mbar_arrive_expect_tx(&idx_full[qs], (uint32_t)p.k * 4u);
          sg_bulk_load(smem + C::OFF_IDX + qs * C::MAX_K * 4, p.indices + it.row * p.k, (uint32_t)p.k * 4u,
                       &idx_full[qs]);
        }
      }
      if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
      const uint16_t* qsrc = p.Q + (it.row * p.Hq + (long long)it.g * 8) * 128;
      const uint32_t qdst = smem_u32(smem + C::OFF_Q + qs * C::SMALL);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int e = lane + 32 * u, h = e >> 4, c = e & 15;  // head h, 16-byte chunk c
        cp_async_16(qdst + (c >> 3) * C::SMALL_PANEL + h * 128 + (((c & 7) ^ h) * 16), qsrc + h * 128 + c * 8, true);
      }
      cp_async_mbar_arrive(&q_full[qs]);
      ++m;
    }
    cp_async_wait<0>();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      // cursor over the CTA's tiles: item, tile j, item ordinal m, tile ordinal n
      long long c_item = blockIdx.x, c_m = 0, c_n = 0;
      int c_j = 0;
      auto skip_to_item = [&](long long& item) {
        SGItem it;
        while (item < n_items && !sg_item(p, item, it)) item += gridDim.x;
      };
      skip_to_item(c_item);
      auto issue_s = [&](long long item_m, int j, long long n) -> bool {
        const int qs = (int)(item_m & 1), ks = (int)(n % C::KS), sb = (int)(n & 1);
        if (j == 0 && !mbar_wait(&q_full[qs], (uint32_t)((item_m >> 1) & 1), abort_flag, 141)) return false;
        if (!mbar_wait(&k_full[ks], (uint32_t)((n / C::KS) & 1), abort_flag, 142)) return false;
        if (!mbar_wait(&s_empty[sb], (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag, 143)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + C::OFF_K + ks * C::TILE_BYTES);
        const uint32_t q_base = smem_u32(smem + C::OFF_Q + qs * C::SMALL);
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base + sb * 16, smem_desc_kmajor(k_base + pn * C::PANEL + kk * 32, 128),
                      smem_desc_kmajor(q_base + pn * C::SMALL_PANEL + kk * 32, 128), C::IDESC_S, (pn | kk) != 0);
        umma_commit(&s_full[sb]);
        umma_commit(&k_empty[ks]);
        if (j == T - 1) umma_commit(&q_empty[qs]);
        return true;
      };
      auto issue_pv = [&](long long item_m, int j, long long n) -> bool {
        const int ob = (int)(item_m & 1), vs = (int)(n % C::VS), pb = (int)(n & 1);
        if (!mbar_wait(&p_full[pb], (uint32_t)((n >> 1) & 1), abort_flag, 144)) return false;
        if (j == 0 && !mbar_wait(&o_empty[ob], (uint32_t)((item_m >> 1) & 1) ^ 1u, abort_flag, 145)) return false;
        if (!mbar_wait(&v_full[vs], (uint32_t)((n / C::VS) & 1), abort_flag, 146)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + C::OFF_V + vs * C::TILE_BYTES);
        const uint32_t p_base = smem_u32(smem + C::OFF_P + pb * C::SMALL);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // 16 slots per step
          umma_bf16(tmem_base + 32 + ob * 16, smem_desc_mn_sw128(v_base + kk * 16 * 128, C::PANEL),
                    smem_desc_kmajor(p_base + (kk >> 2) * C::SMALL_PANEL + (kk & 3) * 32, 128), C::IDESC_O,
                    (j | kk) != 0);
        umma_commit(&v_empty[vs]);
        umma_commit(&p_empty[pb]);
        if (j == T - 1) umma_commit(&o_full[ob]);
        return true;
      };
      if (c_item < n_items) ok = issue_s(c_m, c_j, c_n);
      while (ok && c_item < n_items) {
        // the next tile of the sequence
        long long x_item = c_item, x_m = c_m, x_n = c_n + 1;
        int x_j = c_j + 1;
        if (x_j == T) {
          x_j = 0;
          ++x_m;
          x_item += gridDim.x;
          skip_to_item(x_item);
        }
        if (x_item < n_items && !(ok = issue_s(x_m, x_j, x_n))) break;
        if (!(ok = issue_pv(c_m, c_j, c_n))) break;
        c_item = x_item;
        c_m = x_m;
        c_n = x_n;
        c_j = x_j;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    // Waits are made warp-uniform (__all_sync) and a failed one is carried to the next
    // 128-thread barrier, where the four warps agree on it and leave together: no warp
    // ever leaves while the others wait at a barrier for it.
    const int quarter = warp - 4;
    const int i = quarter * 32 + lane;  // slot of S^T, dimension of O^T
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t p_off = (uint32_t)((i >> 6) * C::SMALL_PANEL + (i & 7) * 2);
    const int pc = (i & 63) >> 3;  // 16-byte chunk of slot i in its P^T row
    long long m = 0, n = 0;
    bool ok = true;
    // (no `ok` in the loop condition: a warp whose last wait failed goes on to the next
    // barrier, where the four warps leave together)
    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
      SGItem it;
      if (!sg_item(p, item, it)) continue;
      const int qs = (int)(m & 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&idx_full[qs], (uint32_t)((m >> 1) & 1), abort_flag, 152)) && ok;
      const int* slots = idx_s + qs * C::MAX_K;
      float mx[8], l[8], r[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        mx[h] = -INFINITY;
        l[h] = 0.f;
        r[h] = 0.f;
      }
      bool left = false;  // the four warps agreed to stop
      for (int j = 0; j < T; ++j, ++n) {
        const int sb = (int)(n & 1);
        const int e = j * 128 + i;
        const int s = (ok && e < p.k) ? slots[e] : -1;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (uint32_t)((n >> 1) & 1), abort_flag, 147)) && ok;
        float x[8];
        if (ok) {
          tc_fence_after();
          tmem_ld_x8_sync(tmem_base + lane_off + sb * 16, x);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        const bool valid = ok && (unsigned)s < (unsigned)it.vis;
        bool up = !ok;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          x[h] = valid ? x[h] * p.scale_log2 : -INFINITY;
          up |= x[h] > mx[h] + 8.f;
        }
        if (named_bar_any(1, 128, up)) {
          // the tile's maxima over the 128 slots; heads whose max moved by more than 8
          float cm[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) cm[h] = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int h = 0; h < 8; ++h) cm[h] = fmaxf(cm[h], __shfl_xor_sync(0xffffffffu, cm[h], o));
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < 8; ++h) red_max[quarter * 8 + h] = cm[h];
            red_ok[quarter] = ok ? 1 : 0;
          }
          named_bar_sync(1, 128);
          if (!(red_ok[0] & red_ok[1] & red_ok[2] & red_ok[3])) {
            ok = false;
            left = true;
            break;  // all four warps
          }
          float alpha[8];
          bool rescale = false;
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const float t = fmaxf(fmaxf(red_max[h], red_max[8 + h]), fmaxf(red_max[16 + h], red_max[24 + h]));
            alpha[h] = 1.f;
            if (t > mx[h] + 8.f) {
              alpha[h] = ex2_ftz(mx[h] - t);  // 0 while the head had no key
              mx[h] = t;
              rescale = true;
            }
            l[h] *= alpha[h];
            r[h] *= alpha[h];
          }
          if (rescale && j > 0) {
            // O^T holds tiles 0..j-1: wait for the last P.V, scale its columns in tensor memory
            const long long q = n - 1;
            ok = __all_sync(0xffffffffu, mbar_wait(&p_empty[q & 1], (uint32_t)((q >> 1) & 1), abort_flag, 148));
            if (ok) {
              tc_fence_after();
              float o[8];
              const uint32_t oaddr = tmem_base + lane_off + 32 + (uint32_t)(m & 1) * 16;
              tmem_ld_x8_sync(oaddr, o);
#pragma unroll
              for (int h = 0; h < 8; ++h) o[h] *= alpha[h];
              tmem_st_x8_sync(oaddr, o);
            }
          }
        }
        float pw[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float mu = mx[h] == -INFINITY ? 0.f : mx[h];
          pw[h] = ex2_ftz(x[h] - mu);
          l[h] += pw[h];
        }
        // P^T operand: row h, slot i (the swizzled K-major layout of the B operand)
        const int pb = (int)(n & 1);
        ok = __all_sync(0xffffffffu, mbar_wait(&p_empty[pb], (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag, 149)) && ok;
        if (ok) {
          uint8_t* pbuf = smem + C::OFF_P + pb * C::SMALL + p_off;
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            const __nv_bfloat16 b = __float2bfloat16_rn(pw[h]);
            r[h] += __bfloat162float(b);
            *reinterpret_cast<__nv_bfloat16*>(pbuf + h * 128 + ((pc ^ h) << 4)) = b;
          }
          fence_proxy_async_shared();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[pb]);
      }
      if (left) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&idx_empty[qs]);  // this warp has read the item's slots
      // ---- the item's sums over its slots, then O = O^T / r
      float v[16];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        v[h] = l[h];
        v[8 + h] = r[h];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] += __shfl_xor_sync(0xffffffffu, v[e], o);
      if (lane == 0) {
#pragma unroll
        for (int e = 0; e < 16; ++e) red_sum[quarter * 16 + e] = v[e];
        red_ok[4 + quarter] = ok ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!(red_ok[4] & red_ok[5] & red_ok[6] & red_ok[7])) {
        ok = false;
        break;  // all four warps
      }
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = (red_sum[e] + red_sum[16 + e]) + (red_sum[32 + e] + red_sum[48 + e]);
      const int ob = (int)(m & 1);
      // a failure here is seen by all four warps at the next item's first barrier
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[ob], (uint32_t)((m >> 1) & 1), abort_flag, 150));
      if (ok) {
        tc_fence_after();
        float o[8];
        tmem_ld_x8_sync(tmem_base + lane_off + 32 + ob * 16, o);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_empty[ob]);
        uint16_t* orow = p.O + (it.row * p.Hq + (long long)it.g * 8) * 128 + i;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          const float inv = v[8 + h] > 0.f ? 1.f / v[8 + h] : 0.f;
          orow[h * 128] = __bfloat16_as_ushort(__float2bfloat16_rn(o[h] * inv));
        }
        if (p.lse && i < 8) {
          float L = 0.f, M = 0.f;
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h == i) {
              L = v[h];
              M = mx[h];
            }
          p.lse[it.row * p.Hq + it.g * 8 + i] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
        }
      }
      ++m;
    }
  } else {
    // ------------------------------------------------------------ K / V copies
    const bool is_v = warp >= 11;
    const int wg = is_v ? warp - 11 : (warp < 4 ? warp - 2 : warp - 6);
    const int nw = is_v ? C::GV : C::GK;
    const int stages = is_v ? C::VS : C::KS;
    uint64_t* full = is_v ? v_full : k_full;
    uint64_t* empty = is_v ? v_empty : k_empty;
    const uint32_t ring = smem_u32(smem + (is_v ? C::OFF_V : C::OFF_K));
    const uint16_t* src = is_v ? p.V : p.K;
    long long n = 0, m = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      SGItem it;
      if (!sg_item(p, item, it)) continue;
      const int qs = (int)(m & 1);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(&idx_full[qs], (uint32_t)((m >> 1) & 1), abort_flag, 153)))) break;
      const int* slots = idx_s + qs * C::MAX_K;
      const uint16_t* base = src + (long long)it.g * 128;
      for (int j = 0; j < T; ++j, ++n) {
        const int st = (int)(n % stages);
        if (lane == 0) ok = mbar_wait(&empty[st], (uint32_t)((n / stages) & 1) ^ 1u, abort_flag, is_v ? 139 : 138);
        if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
        sg_copy_tile(ring + st * C::TILE_BYTES, base, slots + j * 128, p.k - j * 128, it.kbase, it.vis, kv_stride, nw,
                     wg, lane, &full[st]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&idx_empty[qs]);  // the slots are in registers or copies by now
      ++m;
    }
    cp_async_wait<0>();  // nothing of this thread's in flight when the CTA leaves
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

namespace dsa_host {

bool sa_gather_tc_eligible(int Hq, int Hkv, int d, int k, const void* indices) {
  return d == 128 && Hkv > 0 && Hq == 8 * Hkv && k > 0 && k % 16 == 0 && k <= dsa::SGCfg::MAX_K &&
         (reinterpret_cast<uintptr_t>(indices) & 15u) == 0;
}

int sa_gather_tc_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                        const int* cu_k, int batch, long long total_q, int Hq, int Hkv, int k, float scale, void* O,
                        float* lse, cudaStream_t stream, const uint8_t* skip_rows) {
  using C = dsa::SGCfg;
  static DeviceFlag done;
  if (!done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sa_gather_tc_kernel,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    done = true;
  }
  dsa::SGParams p{};
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
  p.k = k;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.O = static_cast<uint16_t*>(O);
  p.lse = lse;
  p.skip_rows = skip_rows;
  const long long n_items = total_q * Hkv;
  if (n_items <= 0) return DSA_OK;
  const long long grid = std::min<long long>(n_items, (long long)sm_count());
  return launch_pdl(false, dsa::sa_gather_tc_kernel, dim3((unsigned)grid), dim3(C::THREADS), (size_t)C::SMEM_BYTES,
                    stream, p);
}

}  // namespace dsa_host
