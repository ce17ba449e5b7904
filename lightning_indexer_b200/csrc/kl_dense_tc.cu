// Dense attention LSE of the KL target on tcgen05 tensor cores (sm_100a).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: the dense warm-up
// trains the indexer against the full attention distribution; its target needs, for every
// query row t and head h, the log-sum-exp of the dense causal logits
//   lse[t,h] = log sum_{s visible to t} exp(scale * Q[t,h] . K[s, h / (Hq/Hkv)]).
//
// One work item is (16 query rows of one sequence, one KV head g): the A operand is the
// 16 rows x 8 query heads of group g (M = 128, read by a 3-D TMA box straight from
// Q [T, Hq, d]), the B operand a tile of 128 keys of K [Tk, Hkv, d] (3-D box, head g),
// K = d = 128.  Each TMEM lane is one (row, head), so the online log-sum-exp over the keys
// is thread-local in the epilogue.  Persistent CTAs, warp-specialised: warp 0 TMA, warp 1
// MMA issuer and TMEM owner, warps 2-5 epilogue; two accumulator buffers, four key stages.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct KlLseParams {
  const int* cu_q;
  const int* cu_k;
  int batch;
  int Hq, Hkv;
  float scale_log2;
  float* lse_out;  // [T, Hq] natural log
  long long n_blocks;  // 16-row blocks over all sequences
  long long n_items;   // n_blocks * Hkv
};

struct KlLseItem {
  long long t0;
  int ntok, i0, Lq, Lk, kbase, g, ntiles;
};

// item -> (block, head); blocks are numbered from the last (usually the longest rows)
__device__ __forceinline__ bool kl_lse_item(long long item, const KlLseParams& p, KlLseItem& it) {
  it.g = (int)(item % p.Hkv);
  long long r = p.n_blocks - 1 - item / p.Hkv;
  for (int b = 0; b < p.batch; ++b) {
    const int Lq = p.cu_q[b + 1] - p.cu_q[b];
    const long long nb = (Lq + 15) / 16;
    if (r < nb) {
      it.i0 = (int)(r * 16);
      it.t0 = p.cu_q[b] + it.i0;
      it.ntok = min(16, Lq - it.i0);
      it.Lq = Lq;
      it.Lk = p.cu_k[b + 1] - p.cu_k[b];
      it.kbase = p.cu_k[b];
      const int vis_last = min(max(it.i0 + it.ntok - 1 + it.Lk - it.Lq + 1, 0), it.Lk);
      it.ntiles = (vis_last + 127) / 128;
      return it.ntiles > 0;
    }
    r -= nb;
  }
  return false;
}

struct KlLseCfg {
  static constexpr int TILE_BYTES = 128 * 128 * 2;
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int B_STAGES = 4;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + TILE_BYTES;
  static constexpr int OFF_BAR = OFF_B + B_STAGES * TILE_BYTES;
  static constexpr int NUM_BARS = 2 + 2 * B_STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int THREADS = 64 + 128;
  static constexpr int TMEM_COLS = 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, 128);
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(KlLseCfg::THREADS, 1)
    kl_lse_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const KlLseParams p) {
  using C = KlLseCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* b_full = bars + 2;                 // [B_STAGES]
  uint64_t* b_empty = bars + 2 + C::B_STAGES;  // [B_STAGES]
  uint64_t* acc_full = bars + 2 + 2 * C::B_STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;               // [2]
  uint64_t* mma_done = acc_full + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < C::B_STAGES; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_q);
    tma_prefetch_desc(&tmap_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int G = p.Hq / p.Hkv;  // 8

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long m = 0, n = 0;  // items, key tiles
      bool ok = true;
      for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        KlLseItem it;
        if (!kl_lse_item(item, p, it)) continue;
        if (!(ok = mbar_wait(a_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 60))) break;
        mbar_arrive_expect_tx(a_full, C::TILE_BYTES);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(sA + pn * C::PANEL_BYTES, &tmap_q, a_full, pn * 64, it.g * G, (int)it.t0);
        ++m;
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int st = (int)(n % C::B_STAGES);
          if (!(ok = mbar_wait(&b_empty[st], (uint32_t)((n / C::B_STAGES) & 1) ^ 1u, abort_flag, 61))) break;
          mbar_arrive_expect_tx(&b_full[st], C::TILE_BYTES);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(sB + st * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmap_k, &b_full[st], pn * 64, it.g,
                        it.kbase + j * 128);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long m = 0, n = 0;
      bool ok = true;
      const uint32_t a_base = smem_u32(sA);
      for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        KlLseItem it;
        if (!kl_lse_item(item, p, it)) continue;
        if (!(ok = mbar_wait(a_full, (uint32_t)(m & 1), abort_flag, 62))) break;
        tc_fence_after();
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int st = (int)(n % C::B_STAGES);
          const int ab = (int)(n & 1);
          if (!(ok = mbar_wait(&acc_empty[ab], (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag, 63))) break;
          if (!(ok = mbar_wait(&b_full[st], (uint32_t)((n / C::B_STAGES) & 1), abort_flag, 64))) break;
          tc_fence_after();
          const uint32_t b_base = smem_u32(sB + st * C::TILE_BYTES);
#pragma unroll
          for (int pn = 0; pn < 2; ++pn)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tmem_base + ab * 128, smem_desc_kmajor(a_base + pn * C::PANEL_BYTES + kk * 32, 128),
                        smem_desc_kmajor(b_base + pn * C::PANEL_BYTES + kk * 32, 128), C::IDESC, (pn | kk) != 0);
          umma_commit(&b_empty[st]);
          umma_commit(&acc_full[ab]);
        }
        if (!ok) break;
        umma_commit(a_empty);
        ++m;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (4 warps)
    const int lane_grp = warp % 4;
    const int r = lane_grp * 32 + lane;  // (row, head) of this thread: row r / 8, head r % 8
    const uint32_t lane_off = (uint32_t)(lane_grp * 32) << 16;
    long long n = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      KlLseItem it;
      if (!kl_lse_item(item, p, it)) continue;
      const int u = r / 8;
      const bool valid = u < it.ntok;
      const int vis = min(max(it.i0 + u + it.Lk - it.Lq + 1, 0), it.Lk);
      float mx = -INFINITY, l = 0.f;
      for (int j = 0; j < it.ntiles; ++j, ++n) {
        const int ab = (int)(n & 1);
        if (!(ok = mbar_wait(&acc_full[ab], (uint32_t)((n >> 1) & 1), abort_flag, 65))) break;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          float v[32];
          tmem_ld_x32_sync(tmem_base + lane_off + ab * 128 + c0, v);
          const int sb = j * 128 + c0;  // first key of the chunk
          float cm = -INFINITY;
#pragma unroll
          for (int q = 0; q < 32; ++q) {
            v[q] = (sb + q < vis) ? v[q] * p.scale_log2 : -INFINITY;
            cm = fmaxf(cm, v[q]);
          }
          if (cm > mx) {
            l *= exp2f(mx - cm);  // mx = -inf: l is 0
            mx = cm;
          }
          if (mx > -INFINITY) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int q = 0; q < 32; q += 2) {
              a0 += exp2f(v[q] - mx);
              a1 += exp2f(v[q + 1] - mx);
            }
            l += a0 + a1;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
      }
      if (!ok) break;
      if (valid)
        p.lse_out[(it.t0 + u) * p.Hq + it.g * G + (r % 8)] =
            l > 0.f ? (mx + log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

namespace dsa_host {

// Dense LSE of every (row, head) for d = 128 and 8 query heads per KV head.
int kl_lse_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                     long long Tk, int Hq, int Hkv, int max_seqlen_q, float scale_log2, float* lse_out,
                     cudaStream_t s) {
  using C = dsa::KlLseCfg;
  static bool attr_done = false;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_lse_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  CUtensorMap tq, tk;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)T};
    const uint64_t strides[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 8, 16};
    if (const int st = make_tmap_bf16_3d(&tq, Q, dims, strides, box); st != DSA_OK) return st;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)Tk};
    const uint64_t strides[2] = {256, (uint64_t)Hkv * 256};
    const uint32_t box[3] = {64, 1, 128};
    if (const int st = make_tmap_bf16_3d(&tk, K, dims, strides, box); st != DSA_OK) return st;
  }
  dsa::KlLseParams p;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.scale_log2 = scale_log2;
  p.lse_out = lse_out;
  // an upper bound on the 16-row blocks (each sequence rounds up once)
  p.n_blocks = (T + 15) / 16 + batch;
  p.n_items = p.n_blocks * Hkv;
  (void)max_seqlen_q;
  const long long grid = std::min<long long>(p.n_items, (long long)sm_count());
  if (grid <= 0) return DSA_OK;
  dsa::kl_lse_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, p);
  return last_launch_status();
}

}  // namespace dsa_host
