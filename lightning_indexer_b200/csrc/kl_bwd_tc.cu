// Indexer backward of the KL loss on tcgen05 tensor cores (sm_100a): the key-stationary
// dk_idx kernel (first below) and the row-stationary dw / dq_idx kernel (second).
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: in the dense warm-up
// only the indexer is trained, by the KL divergence to the full attention distribution.
// With g[t,s] = dloss/dI[t,s] (from the KL target pass) and x[t,j,s] = q_idx[t,j].k_idx[s],
//   dk_idx[s] = sum_t sum_j g[t,s] w[t,j] [x[t,j,s] > 0] q_idx[t,j,:].
//
// One work item is (sequence, tile of 128 keys, block of up to KL_DK_ROWS query rows of the
// row chunk that see the tile).  The items of a chunk are counted on the device (a prefix
// sum over (sequence, tile) pairs), so their partial dk (128 keys x d_I, fp32) sit in one
// compact slot each, and a second kernel adds a tile's slots in item order (deterministic).
// Small items keep the persistent CTAs evenly loaded on chunks of short sequences.
// Per block of 2 query rows (N = 2 x 64 heads = 128 columns), two chained MMAs:
//   MMA1  X[128 keys x 128 (t,j)] = K_tile . Q_blk^T          (TMEM, two buffers)
//   epilogue  G = g w [X > 0] -> bf16, written to shared memory in the 128-byte swizzled
//             K-major layout the tensor core reads (row = key, 16-byte chunk c of a row
//             at chunk c ^ (row % 8))
//   MMA2  dk[128 keys x 128 d] += G . Q_blk                   (TMEM accumulator)
// MMA2's B operand is the same query block read MN-major (d contiguous), so the block is
// loaded once for both MMAs.
// MMA1 of the next block is issued before MMA2 of this one, so the tensor pipe computes X
// while the epilogue turns the previous X into G.  Warp roles: warp 0 TMA producer, warp 1
// MMA issuer and TMEM owner, warps 2-9 epilogue (one TMEM lane, i.e. one key, per thread;
// two warps per lane quarter, one per query row of the block).
#include <algorithm>
#include <type_traits>

#include "common.cuh"

namespace dsa {

// query rows per dk work item (a multiple of 2)
constexpr int KL_DK_ROWS = 256;
// (sequence, tile) pairs whose item offsets are cached in shared memory
constexpr int KL_DK_SMEM_PAIRS = 4095;

// rows [qlo, qhi) of the chunk [row_begin, row_end) that see key tile `tile` of sequence b
__device__ __forceinline__ void dk_tile_rows(const int* cu_q, const int* cu_k, int b, int tile, long long row_begin,
                                             long long row_end, long long& qlo, long long& qhi) {
  const int Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
  qlo = max((long long)cu_q[b] + max(tile * 128 - (Lk - Lq), 0), row_begin);
  qhi = min((long long)cu_q[b + 1], row_end);
  if (tile * 128 >= Lk) qhi = qlo;
}

// offs[pair] = first item of (sequence, tile) pair = b * tiles_per_seq + tile, offs[n_pairs]
// = the chunk's item count (one block; exclusive scan in rounds of blockDim.x pairs)
__global__ void dk_items_kernel(const int* cu_q, const int* cu_k, int batch, int tiles_per_seq, long long row_begin,
                                long long row_end, int* offs) {
  __shared__ int warp_sums[32];
  __shared__ int carry;
  const long long n_pairs = (long long)batch * tiles_per_seq;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (long long base = 0; base < n_pairs; base += blockDim.x) {
    const long long pr = base + threadIdx.x;
    int cnt = 0;
    if (pr < n_pairs) {
      long long qlo, qhi;
      dk_tile_rows(cu_q, cu_k, (int)(pr / tiles_per_seq), (int)(pr % tiles_per_seq), row_begin, row_end, qlo, qhi);
      cnt = qhi > qlo ? (int)((qhi - qlo + KL_DK_ROWS - 1) / KL_DK_ROWS) : 0;
    }
    // inclusive warp scan, then across warps
    int v = cnt;
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane == 31) warp_sums[wid] = v;
    __syncthreads();
    if (wid == 0) {
      int ws = lane < (int)(blockDim.x / 32) ? warp_sums[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, ws, o);
        if (lane >= o) ws += y;
      }
      warp_sums[lane] = ws;
    }
    __syncthreads();
    const int before = carry + (wid > 0 ? warp_sums[wid - 1] : 0) + v - cnt;
    if (pr < n_pairs) offs[pr] = before;
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) carry = before + cnt;
    __syncthreads();
  }
  if (threadIdx.x == 0) offs[n_pairs] = carry;
}

// dk_acc[key] += the slots of key's (sequence, tile) pair, in item order (one thread per 4
// consecutive values of one key)
__global__ void dk_reduce_items_kernel(const float* __restrict__ dk_part, const int* __restrict__ offs,
                                       int tiles_per_seq, const int* cu_k, int batch, long long Tk, float* dk_acc) {
  const long long e = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (e >= Tk * 128) return;
  const long long key = e / 128;
  const int c = (int)(e % 128);
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)cu_k[mid] <= key) lo = mid; else hi = mid;
  }
  const int sl = (int)(key - cu_k[lo]);
  const int pair = lo * tiles_per_seq + sl / 128, r = sl % 128;
  const int i0 = offs[pair], i1 = offs[pair + 1];
  if (i0 == i1) return;
  float4 acc = *reinterpret_cast<const float4*>(dk_acc + e);
  for (int i = i0; i < i1; ++i) {
    const float4 v = *reinterpret_cast<const float4*>(dk_part + ((size_t)i * 128 + r) * 128 + c);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  *reinterpret_cast<float4*>(dk_acc + e) = acc;
}

struct KlDkParams {
  const uint16_t* w;  // [T, 64] bf16
  long long total_q;
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin, row_end;  // the row chunk
  const float* g;                // [row_end - row_begin, ld] fp32 dloss/dI
  long long ld;
  int tiles_per_seq;
  int n_pairs;                   // batch * tiles_per_seq
  const int* offs;               // [n_pairs + 1] first item of each pair (dk_items_kernel)
  float* dk_part;                // [items][128 keys][128] fp32
};

struct KlDkItem {
  long long slot;      // partial slot (the item index)
  int b, tile, kbase, Lq, Lk;
  long long qlo, qhi;  // the item's query rows
  int nb;              // blocks of 2 rows
};

// item index -> (pair, row block) by a search over the pair offsets `offs` (shared or global)
__device__ __forceinline__ void kl_dk_item(long long item, const KlDkParams& p, const int* offs, KlDkItem& it) {
  int lo = 0, hi = p.n_pairs;  // offs[lo] <= item < offs[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (offs[mid] <= item) lo = mid; else hi = mid;
  }
  const int b = lo / p.tiles_per_seq, tile = lo % p.tiles_per_seq;
  long long qlo, qhi;
  dk_tile_rows(p.cu_q, p.cu_k, b, tile, p.row_begin, p.row_end, qlo, qhi);
  qlo += (item - offs[lo]) * KL_DK_ROWS;
  qhi = min(qhi, qlo + KL_DK_ROWS);
  it.slot = item;
  it.b = b;
  it.tile = tile;
  it.kbase = p.cu_k[b];
  it.Lq = p.cu_q[b + 1] - p.cu_q[b];
  it.Lk = p.cu_k[b + 1] - it.kbase;
  it.qlo = qlo;
  it.qhi = qhi;
  it.nb = (int)((qhi - qlo + 1) / 2);
}

struct KlDkCfg {
  static constexpr int H_I = 64, D_I = 128, NTOK = 2, N = NTOK * H_I;  // 128 columns
  static constexpr int TILE_BYTES = 128 * 128 * 2;                      // any 128 x 128 bf16 operand
  static constexpr int PANEL_BYTES = 128 * 128;                         // 128 rows x 128 B
  static constexpr int Q_STAGES = 3;
  static constexpr int OFF_A = 0;                                       // key tile
  static constexpr int OFF_Q = OFF_A + TILE_BYTES;                      // Q_STAGES x Q_blk
  static constexpr int OFF_G = OFF_Q + Q_STAGES * TILE_BYTES;           // 2 G buffers
  static constexpr int OFF_W = OFF_G + 2 * TILE_BYTES;                  // Q_STAGES x w of the block's rows
  static constexpr int W_BYTES = 2 * 64 * 2;
  static constexpr int OFF_GS = OFF_W + Q_STAGES * W_BYTES;            // Q_STAGES x g of the block's rows
  static constexpr int GS_BYTES = 2 * 128 * 4;
  static constexpr int OFF_OFFS = OFF_GS + Q_STAGES * GS_BYTES;       // cached item offsets
  static constexpr int OFF_BAR = OFF_OFFS + (KL_DK_SMEM_PAIRS + 1) * 4;
  // a_full, a_empty, q_full[S], q_empty[S], x_full[2], x_empty[2], g_full[2], g_empty[2],
  // dk_full, dk_empty, done
  static constexpr int NUM_BARS = 2 + 2 * Q_STAGES + 8 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int EPI_WARPS = 8;  // two per TMEM lane quarter: one per block row (64 columns)
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int TMEM_COLS = 512;  // X buffers [0,128) [128,256), dk [256,384)
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, 128);
  static constexpr uint32_t IDESC2 = idesc_bf16_f32(128, 128) | kIdescBMnMajor;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(KlDkCfg::THREADS, 1)
    kl_dk_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                    const KlDkParams p) {
  using C = KlDkCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sG = smem + C::OFF_G;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + 1;
  uint64_t* q_full = bars + 2;                  // [Q_STAGES]
  uint64_t* q_empty = q_full + C::Q_STAGES;     // [Q_STAGES]
  uint64_t* x_full = q_empty + C::Q_STAGES;     // [2]
  uint64_t* x_empty = x_full + 2;               // [2]
  uint64_t* g_full = x_full + 4;                // [2]
  uint64_t* g_empty = x_full + 6;               // [2]
  uint64_t* dk_full = x_full + 8;
  uint64_t* dk_empty = x_full + 9;
  uint64_t* mma_done = x_full + 10;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < C::Q_STAGES; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], C::EPI_WARPS);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&g_full[i], C::EPI_WARPS);
      mbar_init(&g_empty[i], 1);
    }
    mbar_init(dk_full, 1);
    mbar_init(dk_empty, C::EPI_WARPS);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  // the chunk's item offsets: shared-memory copy when they fit
  int* s_offs = reinterpret_cast<int*>(smem + C::OFF_OFFS);
  const bool offs_in_smem = p.n_pairs <= KL_DK_SMEM_PAIRS;
  if (offs_in_smem)
    for (int i = threadIdx.x; i <= p.n_pairs; i += blockDim.x) s_offs[i] = p.offs[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int* offs = offs_in_smem ? s_offs : p.offs;
  const long long n_items = offs[p.n_pairs];
  const long long n_slots = (n_items + gridDim.x - 1) / gridDim.x * gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long n = 0;  // blocks loaded so far (stage n % Q_STAGES)
      long long m = 0;  // non-empty items so far
      bool ok = true;
      for (long long slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
        const long long item = snake_slot(slot);
        if (item >= n_items) continue;
        KlDkItem it;
        kl_dk_item(item, p, offs, it);
        if (!(ok = mbar_wait(a_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 40))) break;
        mbar_arrive_expect_tx(a_full, C::TILE_BYTES);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_2d(sA + pn * C::PANEL_BYTES, &tmap_k, a_full, pn * 64, it.kbase + it.tile * 128);
        ++m;
        for (int i = 0; i < it.nb; ++i, ++n) {
          const int st = (int)(n % C::Q_STAGES);
          if (!(ok = mbar_wait(&q_empty[st], (uint32_t)((n / C::Q_STAGES) & 1) ^ 1u, abort_flag, 41))) break;
          const long long t0 = it.qlo + 2 * i;
          // head weights of the block's rows that exist in the tensor (the second may not)
          const uint32_t wbytes = (uint32_t)(min(2LL, p.total_q - t0) * C::H_I * 2);
          // g of the block's rows in the item for the tile's keys (rows end at ld; ld % 4 == 0)
          const int grows = (int)min(2LL, it.qhi - t0);
          const uint32_t gbytes = (uint32_t)(min(128LL, p.ld - (long long)it.tile * 128) * 4);
          mbar_arrive_expect_tx(&q_full[st], C::TILE_BYTES + wbytes + grows * gbytes);
          uint8_t* sq = sQ + st * C::TILE_BYTES;
          const int col = (int)(t0 * C::H_I);  // first (t, j) row of the block
          for (int pn = 0; pn < 2; ++pn) tma_load_2d(sq + pn * C::PANEL_BYTES, &tmap_q, &q_full[st], pn * 64, col);
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_u32(smem + C::OFF_W + st * C::W_BYTES)),
              "l"(p.w + t0 * C::H_I), "r"(wbytes), "r"(smem_u32(&q_full[st]))
              : "memory");
          for (int r = 0; r < grows; ++r)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                    smem_u32(smem + C::OFF_GS + st * C::GS_BYTES + r * 512)),
                "l"(p.g + (t0 + r - p.row_begin) * p.ld + (long long)it.tile * 128), "r"(gbytes),
                "r"(smem_u32(&q_full[st]))
                : "memory");
        }
      }
      if (!ok) {
        // drain: the loads this thread issued land before the CTA can exit
        const uint64_t t0 = globaltimer_ns();
        for (long long k = max(0LL, n - C::Q_STAGES); k < n; ++k)
          while (!mbar_try_wait(smem_u32(&q_full[k % C::Q_STAGES]), (uint32_t)((k / C::Q_STAGES) & 1)) &&
                 globaltimer_ns() - t0 < 200000000ull) {
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long n = 0;  // blocks whose MMA1 was issued
      long long m = 0;  // non-empty items
      long long gcount = 0;
      bool ok = true;
      const uint32_t a_base = smem_u32(sA);
      const uint32_t g_base = smem_u32(sG);
      const uint32_t dk_tmem = tmem_base + 256;
      auto mma1 = [&](long long blk) -> bool {
        const int st = (int)(blk % C::Q_STAGES), xb = (int)(blk & 1);
        if (!mbar_wait(&q_full[st], (uint32_t)((blk / C::Q_STAGES) & 1), abort_flag, 42)) return false;
        if (!mbar_wait(&x_empty[xb], (uint32_t)((blk >> 1) & 1) ^ 1u, abort_flag, 43)) return false;
        tc_fence_after();
        const uint32_t q_base = smem_u32(sQ + st * C::TILE_BYTES);
        const uint32_t d_tmem = tmem_base + xb * 128;
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(d_tmem, smem_desc_kmajor(a_base + pn * C::PANEL_BYTES + kk * 32, 128),
                      smem_desc_kmajor(q_base + pn * C::PANEL_BYTES + kk * 32, 128), C::IDESC, (pn | kk) != 0);
        umma_commit(&x_full[xb]);
        return true;
      };
      for (long long slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
        const long long item = snake_slot(slot);
        if (item >= n_items) continue;
        KlDkItem it;
        kl_dk_item(item, p, offs, it);
        if (!(ok = mbar_wait(a_full, (uint32_t)(m & 1), abort_flag, 44))) break;
        tc_fence_after();
        const long long n0 = n;
        if (!(ok = mma1(n))) break;
        ++n;
        for (int i = 0; i < it.nb && ok; ++i) {
          if (i + 1 < it.nb) {
            if (!(ok = mma1(n))) break;
            ++n;
          }
          if (i + 1 == it.nb) umma_commit(a_empty);  // the key tile is free once these MMAs finish
          const int gb = (int)(gcount & 1);
          if (!(ok = mbar_wait(&g_full[gb], (uint32_t)((gcount >> 1) & 1), abort_flag, 45))) break;
          if (i == 0 && !(ok = mbar_wait(dk_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 46))) break;
          tc_fence_after();
          const long long blk = n0 + i;
          const int qs = (int)(blk % C::Q_STAGES);
          const uint32_t q_base = smem_u32(sQ + qs * C::TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 (t,j) rows of the block per step
            umma_bf16(dk_tmem,
                      smem_desc_kmajor(g_base + gb * C::TILE_BYTES + (kk / 4) * C::PANEL_BYTES + (kk % 4) * 32, 128),
                      smem_desc_mn_sw128(q_base + kk * 16 * 128, C::PANEL_BYTES), C::IDESC2, (i | kk) != 0);
          umma_commit(&g_empty[gb]);
          umma_commit(&q_empty[qs]);
          ++gcount;
        }
        if (!ok) break;
        umma_commit(dk_full);
        ++m;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int lane_grp = warp % 4;             // TMEM lane quarter this warp may access
    const int half = (warp - 2) / 4;           // block row (and column half) of this warp
    const int r = lane_grp * 32 + lane;        // key row of this thread within the tile
    const uint32_t lane_off = (uint32_t)(lane_grp * 32) << 16;
    const uint32_t g_row0 = smem_u32(sG) + half * C::PANEL_BYTES + r * 128;
    long long n = 0, m = 0, gcount = 0;
    bool ok = true;
    for (long long slot = blockIdx.x; slot < n_slots && ok; slot += gridDim.x) {
      const long long item = snake_slot(slot);
      if (item >= n_items) continue;
      KlDkItem it;
      kl_dk_item(item, p, offs, it);
      const int s = it.tile * 128 + r;  // this thread's key (sequence-local)
      const int dvis = it.Lk - it.Lq + 1;
      const long long q0 = p.cu_q[it.b];
      for (int i = 0; i < it.nb; ++i, ++n) {
        const long long t = it.qlo + 2 * i + half;  // this warp's query row
        // its G columns are 0 past the item or the row's visible keys
        const bool tv = t < it.qhi && s < min(max((int)(t - q0) + dvis, 0), it.Lk);
        const int st = (int)(n % C::Q_STAGES), xb = (int)(n & 1);
        // the block's head weights arrive with its query tile: observe that phase here too
        // (the stage cannot be refilled before this block's G is written, so the phase seen
        // is this block's)
        if (!(ok = mbar_wait(&q_full[st], (uint32_t)((n / C::Q_STAGES) & 1), abort_flag, 50))) break;
        const uint4* sW = reinterpret_cast<const uint4*>(smem + C::OFF_W + st * C::W_BYTES + half * C::H_I * 2);
        const float gv = tv ? reinterpret_cast<const float*>(smem + C::OFF_GS + st * C::GS_BYTES)[half * 128 + r] : 0.f;
        if (!(ok = mbar_wait(&x_full[xb], (uint32_t)((n >> 1) & 1), abort_flag, 47))) break;
        tc_fence_after();
        float x[64];
        tmem_ld_x32_sync(tmem_base + lane_off + xb * 128 + half * 64, x);
        tmem_ld_x32_sync(tmem_base + lane_off + xb * 128 + half * 64 + 32, x + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_empty[xb]);
        // G buffer gb may be overwritten once the MMA2 that read it two blocks ago is done
        const int gb = (int)(gcount & 1);
        if (!(ok = mbar_wait(&g_empty[gb], (uint32_t)((gcount >> 1) & 1) ^ 1u, abort_flag, 48))) break;
        const uint32_t g_row = g_row0 + gb * C::TILE_BYTES;
#pragma unroll
        for (int q = 0; q < 8; ++q) {  // 16-byte chunk q of this row's panel: columns 8q .. 8q+7
          uint32_t pk[4];
          const uint4 w8 = sW[q];  // head weights of columns 8q .. 8q+7
          const uint32_t wp[4] = {w8.x, w8.y, w8.z, w8.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = q * 8 + 2 * e;
            const float v0 = x[c] > 0.f ? gv * __uint_as_float(wp[e] << 16) : 0.f;
            const float v1 = x[c + 1] > 0.f ? gv * __uint_as_float(wp[e] & 0xFFFF0000u) : 0.f;
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
            pk[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(g_row + ((q ^ (r & 7)) * 16)),
                       "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                       : "memory");
        }
        fence_proxy_async_shared();  // the tensor core reads G through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&g_full[gb]);
        ++gcount;
      }
      if (!ok) break;
      // the item's dk: one key row per thread, this warp's 64 of its 128 fp32 values
      if (!(ok = mbar_wait(dk_full, (uint32_t)(m & 1), abort_flag, 49))) break;
      tc_fence_after();
      float* dst = p.dk_part + ((size_t)it.slot * 128 + r) * C::D_I + half * 64;
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld_x32_sync(tmem_base + lane_off + 256 + half * 64 + c, v);
        if (s < it.Lk) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c + e) = make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dk_empty);
      ++m;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------- rows
// Row-stationary half of the same backward (H_I = 64, d_I = 128):
//   dw[t,j]     = sum_s g[t,s] max(0, x[t,j,s])
//   dq_idx[t,j] = sum_s g[t,s] w[t,j] [x[t,j,s] > 0] k_idx[s]
// Both come from one product: with u[t,j] = sum_s g[t,s] [x[t,j,s] > 0] k_idx[s],
// dq_idx = w u, and since x is linear in q_idx, dw = sum_s g [x > 0] (q_idx . k_idx[s])
// = q_idx[t,j] . u[t,j], a 128-term dot per (t,j) instead of a term per key.
// One work item is 2 query rows of one sequence of the row chunk (M = 2 x 64 (t,j) pairs
// = 128 TMEM lanes); the item's key tiles of 128 stream through three stages, each with
// the g values of its two rows.  Per key tile:
//   MMA1  X[128 (t,j) x 128 keys] = Q_blk . K_tile^T       (TMEM, two buffers)
//   epilogue  G = g [X > 0] -> bf16 in the 128-byte swizzled K-major layout (K = keys)
//   MMA2  u[128 (t,j) x 128 d] += G . K_tile              (TMEM accumulator)
// and per item dq_idx = w u, dw = q_idx . u (one (t,j) per TMEM lane).
// MMA2's B operand is the key tile itself read MN-major (d contiguous), so no transposed
// copy of k_idx is needed.  MMA1 of the next tile is issued before MMA2 of this one.
// Warps: 0 TMA, 1 MMA issuer and TMEM owner, 2-9 epilogue (two per lane quarter, one per
// 64-key half of the tile; the two dw halves meet in shared memory, added in a fixed order).
struct KlDqParams {
  const uint16_t* q_idx;  // [T, 64, 128] bf16
  const uint16_t* w;      // [T, 64] bf16
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin, row_end;  // the row chunk
  const float* g;                // [row_end - row_begin, ld] fp32 dloss/dI
  long long ld;
  uint16_t* dq;  // [T, 64, 128] bf16
  uint16_t* dw;  // [T, 64] bf16
  long long n_blocks, n_slots;
};

struct KlDqItem {
  long long t0;
  int ntok, i0, Lq, Lk, kbase, ntiles;
};

__device__ __forceinline__ bool kl_dq_item(long long slot, const KlDqParams& p, KlDqItem& it) {
  RowBlock rb;
  if (!chunk_row_block<2>(snake_slot(slot), p.cu_q, p.cu_k, p.batch, p.row_begin, p.row_end, p.n_blocks, rb))
    return false;
  it.t0 = rb.t0;
  it.ntok = rb.ntok;
  it.i0 = rb.i0;
  it.Lq = rb.Lq;
  it.Lk = rb.Lk;
  it.kbase = rb.kbase;
  it.ntiles = (causal_vis(it.i0 + it.ntok - 1, it.Lq, it.Lk) + 127) / 128;
  return true;
}

struct KlDqCfg {
  static constexpr int H_I = 64, D_I = 128;
  static constexpr int TILE_BYTES = 128 * 128 * 2;
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int K_STAGES = 3;
  static constexpr int GS_BYTES = 2 * 128 * 4;  // g of the 2 rows for one key tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_G = OFF_K + K_STAGES * TILE_BYTES;  // 2 G buffers
  static constexpr int OFF_GS = OFF_G + 2 * TILE_BYTES;
  static constexpr int OFF_DW = OFF_GS + K_STAGES * GS_BYTES;  // 128 fp32 dw halves
  static constexpr int OFF_BAR = OFF_DW + 128 * 4;
  // q_full, q_empty, k_full[S], k_empty[S], x_full[2], x_empty[2], g_full[2], g_empty[2],
  // dq_full, dq_empty, dw_full, dw_empty, done
  static constexpr int NUM_BARS = 2 + 2 * K_STAGES + 8 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int TMEM_COLS = 512;  // X buffers [0,128) [128,256), dq [256,384)
  static constexpr uint32_t IDESC1 = idesc_bf16_f32(128, 128);
  static constexpr uint32_t IDESC2 = idesc_bf16_f32(128, 128) | kIdescBMnMajor;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(KlDqCfg::THREADS, 1)
    kl_dq_tc_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                    const KlDqParams p) {
  using C = KlDqCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sG = smem + C::OFF_G;
  float* sGs = reinterpret_cast<float*>(smem + C::OFF_GS);
  float* sDw = reinterpret_cast<float*>(smem + C::OFF_DW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                 // [K_STAGES]
  uint64_t* k_empty = k_full + C::K_STAGES;    // [K_STAGES]
  uint64_t* x_full = k_empty + C::K_STAGES;    // [2]
  uint64_t* x_empty = x_full + 2;              // [2]
  uint64_t* g_full = x_full + 4;               // [2]
  uint64_t* g_empty = x_full + 6;              // [2]
  uint64_t* dq_full = x_full + 8;
  uint64_t* dq_empty = x_full + 9;
  uint64_t* dw_full = x_full + 10;
  uint64_t* dw_empty = x_full + 11;
  uint64_t* mma_done = x_full + 12;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::K_STAGES; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], C::EPI_WARPS);
      mbar_init(&g_full[i], C::EPI_WARPS);
      mbar_init(&g_empty[i], 1);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, C::EPI_WARPS);
    mbar_init(dw_full, C::EPI_WARPS / 2);
    mbar_init(dw_empty, C::EPI_WARPS / 2);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long m = 0, n = 0;  // items with key tiles, key tiles
      bool ok = true;
      for (long long slot = blockIdx.x; slot < p.n_slots && ok; slot += gridDim.x) {
        KlDqItem it;
        if (!kl_dq_item(slot, p, it) || it.ntiles == 0) continue;
        if (!(ok = mbar_wait(q_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 80))) break;
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_2d(sQ + pn * C::PANEL_BYTES, &tmap_q, q_full, pn * 64, (int)(it.t0 * C::H_I));
        ++m;
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int st = (int)(n % C::K_STAGES);
          if (!(ok = mbar_wait(&k_empty[st], (uint32_t)((n / C::K_STAGES) & 1) ^ 1u, abort_flag, 81))) break;
          // g of the block's rows for this tile's keys (the row ends at ld; ld % 4 == 0)
          const uint32_t gbytes = (uint32_t)(min(128LL, p.ld - (long long)j * 128) * 4);
          mbar_arrive_expect_tx(&k_full[st], C::TILE_BYTES + it.ntok * gbytes);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_2d(sK + st * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmap_k, &k_full[st], pn * 64,
                        it.kbase + j * 128);
          for (int r = 0; r < it.ntok; ++r)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                    smem_u32(sGs + st * (C::GS_BYTES / 4) + r * 128)),
                "l"(p.g + (it.t0 + r - p.row_begin) * p.ld + (long long)j * 128), "r"(gbytes),
                "r"(smem_u32(&k_full[st]))
                : "memory");
        }
      }
      if (!ok) {
        // let the copies this thread issued land before the CTA exits (bounded)
        const uint64_t t0 = globaltimer_ns();
        for (long long k = max(0LL, n - C::K_STAGES); k < n; ++k)
          while (!mbar_try_wait(smem_u32(&k_full[k % C::K_STAGES]), (uint32_t)((k / C::K_STAGES) & 1)) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        if (m > 0)
          while (!mbar_try_wait(smem_u32(q_full), (uint32_t)((m - 1) & 1)) && globaltimer_ns() - t0 < 100000000ull) {
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long m = 0, n = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t g_base = smem_u32(sG);
      const uint32_t dq_tmem = tmem_base + 256;
      auto mma1 = [&](long long u) -> bool {
        const int st = (int)(u % C::K_STAGES), xb = (int)(u & 1);
        if (!mbar_wait(&k_full[st], (uint32_t)((u / C::K_STAGES) & 1), abort_flag, 82)) return false;
        if (!mbar_wait(&x_empty[xb], (uint32_t)((u >> 1) & 1) ^ 1u, abort_flag, 83)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + st * C::TILE_BYTES);
#pragma unroll
        for (int pn = 0; pn < 2; ++pn)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem_base + xb * 128, smem_desc_kmajor(q_base + pn * C::PANEL_BYTES + kk * 32, 128),
                      smem_desc_kmajor(k_base + pn * C::PANEL_BYTES + kk * 32, 128), C::IDESC1, (pn | kk) != 0);
        umma_commit(&x_full[xb]);
        return true;
      };
      auto mma2 = [&](long long u, bool first) -> bool {
        const int st = (int)(u % C::K_STAGES), gb = (int)(u & 1);
        if (!mbar_wait(&g_full[gb], (uint32_t)((u >> 1) & 1), abort_flag, 84)) return false;
        if (first && !mbar_wait(dq_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 85)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_u32(sK + st * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // 16 keys per step
          umma_bf16(dq_tmem,
                    smem_desc_kmajor(g_base + gb * C::TILE_BYTES + (kk / 4) * C::PANEL_BYTES + (kk % 4) * 32, 128),
                    smem_desc_mn_sw128(k_base + kk * 16 * 128, C::PANEL_BYTES), C::IDESC2, !(first && kk == 0));
        umma_commit(&k_empty[st]);
        umma_commit(&g_empty[gb]);
        return true;
      };
      for (long long slot = blockIdx.x; slot < p.n_slots && ok; slot += gridDim.x) {
        KlDqItem it;
        if (!kl_dq_item(slot, p, it) || it.ntiles == 0) continue;
        if (!(ok = mbar_wait(q_full, (uint32_t)(m & 1), abort_flag, 86))) break;
        tc_fence_after();
        for (int j = 0; j < it.ntiles && ok; ++j) {
          if (!(ok = mma1(n + j))) break;
          if (j + 1 == it.ntiles) umma_commit(q_empty);  // the query block is free after these
          if (j > 0 && !(ok = mma2(n + j - 1, j == 1))) break;
        }
        if (!ok) break;
        if (!(ok = mma2(n + it.ntiles - 1, it.ntiles == 1))) break;
        umma_commit(dq_full);
        n += it.ntiles;
        ++m;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quarter = warp % 4;          // TMEM lane quarter: rows 32 quarter .. of the block
    const int half = (warp - 2) / 4;       // keys 64 half .. 64 half + 63 of each tile
    const int mrow = quarter * 32 + lane;  // (t,j) row of the block: t = t0 + mrow / 64
    const int rsel = quarter >> 1;
    const int head = mrow % 64;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t g_row0 = smem_u32(sG) + half * C::PANEL_BYTES + mrow * 128;
    long long m = 0, n = 0;
    bool ok = true;
    for (long long slot = blockIdx.x; slot < p.n_slots && ok; slot += gridDim.x) {
      KlDqItem it;
      if (!kl_dq_item(slot, p, it)) continue;
      const long long t = it.t0 + rsel;
      const bool tv = rsel < it.ntok;
      uint16_t* dq_dst = p.dq + ((size_t)t * C::H_I + head) * C::D_I + half * 64;
      if (it.ntiles == 0) {  // no visible key: dq = 0, dw = 0
        if (tv) {
#pragma unroll
          for (int e = 0; e < 64; e += 8) *reinterpret_cast<uint4*>(dq_dst + e) = make_uint4(0u, 0u, 0u, 0u);
          if (half == 0) p.dw[t * C::H_I + head] = 0;
        }
        continue;
      }
      const int vis = tv ? causal_vis(it.i0 + rsel, it.Lq, it.Lk) : 0;
      const float wv = tv ? bf16_bits_to_f32(p.w[t * C::H_I + head]) : 0.f;
      for (int j = 0; j < it.ntiles; ++j, ++n) {
        const int st = (int)(n % C::K_STAGES), xb = (int)(n & 1);
        // the tile's g values arrive with its keys
        if (!(ok = mbar_wait(&k_full[st], (uint32_t)((n / C::K_STAGES) & 1), abort_flag, 87))) break;
        if (!(ok = mbar_wait(&x_full[xb], (uint32_t)((n >> 1) & 1), abort_flag, 88))) break;
        tc_fence_after();
        float x[64];
        tmem_ld_x32_sync(tmem_base + lane_off + xb * 128 + half * 64, x);
        tmem_ld_x32_sync(tmem_base + lane_off + xb * 128 + half * 64 + 32, x + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&x_empty[xb]);
        const float* gs = sGs + st * (C::GS_BYTES / 4) + rsel * 128 + half * 64;
        const int s0 = j * 128 + half * 64;
        const int nvis = vis - s0;  // keys of this half the row sees (all 64 unless at its end)
        if (!(ok = mbar_wait(&g_empty[xb], (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag, 89))) break;
        const uint32_t g_row = g_row0 + xb * C::TILE_BYTES;
        // G = g [x > 0]; keys past the row's visible ones (only in its last tile) give 0
        auto write_g = [&](auto masked) {
#pragma unroll
          for (int q = 0; q < 8; ++q) {  // 16-byte chunk q of this row's panel: keys 8q .. 8q+7
            const float4 ga = *reinterpret_cast<const float4*>(gs + q * 8);
            const float4 gb = *reinterpret_cast<const float4*>(gs + q * 8 + 4);
            const float gq[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = q * 8 + 2 * e;
              bool k0 = x[c] > 0.f, k1 = x[c + 1] > 0.f;
              if constexpr (decltype(masked)::value) {
                k0 = k0 && c < nvis;
                k1 = k1 && c + 1 < nvis;
              }
              __nv_bfloat162 b2 = __floats2bfloat162_rn(k0 ? gq[2 * e] : 0.f, k1 ? gq[2 * e + 1] : 0.f);
              pk[e] = *reinterpret_cast<uint32_t*>(&b2);
            }
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(g_row + ((q ^ (mrow & 7)) * 16)),
                         "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                         : "memory");
          }
        };
        if (nvis >= 64)
          write_g(std::false_type{});
        else
          write_g(std::true_type{});
        fence_proxy_async_shared();  // the tensor core reads G through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(&g_full[xb]);
      }
      if (!ok) break;
      // u of this thread's (t,j), 64 of its 128 columns: dq_idx = w u (bf16), dw part = q_idx . u
      if (!(ok = mbar_wait(dq_full, (uint32_t)(m & 1), abort_flag, 90))) break;
      tc_fence_after();
      float dw = 0.f;
      const uint4* qrow = reinterpret_cast<const uint4*>(p.q_idx + ((size_t)t * C::H_I + head) * C::D_I + half * 64);
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld_x32_sync(tmem_base + lane_off + 256 + half * 64 + c, v);
        if (tv) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            const uint4 q8 = qrow[(c + e) / 8];
            const uint32_t qp[4] = {q8.x, q8.y, q8.z, q8.w};
            uint4 o;
            uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const float u0 = v[e + 2 * f], u1 = v[e + 2 * f + 1];
              dw = fmaf(__uint_as_float(qp[f] << 16), u0, dw);
              dw = fmaf(__uint_as_float(qp[f] & 0xFFFF0000u), u1, dw);
              __nv_bfloat162 b2 = __floats2bfloat162_rn(wv * u0, wv * u1);
              po[f] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(dq_dst + c + e) = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_empty);
      // dw = (d 0..63 half) + (d 64..127 half), added in this order
      if (half == 1) {
        if (!(ok = mbar_wait(dw_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 91))) break;
        sDw[mrow] = dw;
        __syncwarp();
        if (lane == 0) mbar_arrive(dw_full);
      } else {
        if (!(ok = mbar_wait(dw_full, (uint32_t)(m & 1), abort_flag, 92))) break;
        const float total = dw + sDw[mrow];
        __syncwarp();
        if (lane == 0) mbar_arrive(dw_empty);
        if (tv) {
          __nv_bfloat16 b = __float2bfloat16_rn(total);
          p.dw[t * C::H_I + head] = *reinterpret_cast<uint16_t*>(&b);
        }
      }
      ++m;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

namespace dsa_host {

// Upper bound on the dk work items of one row chunk: every item but the last of each
// (sequence, tile) pair covers KL_DK_ROWS rows of the chunk.
size_t kl_dk_tc_max_items(long long chunk_rows, long long total_k, int batch, int max_seqlen_k) {
  const long long tiles = (max_seqlen_k + 127) / 128;
  return (size_t)((total_k + 127) / 128 + batch + (chunk_rows * tiles + dsa::KL_DK_ROWS - 1) / dsa::KL_DK_ROWS);
}

// dk_acc += dk of the row chunk [r0, r1) for H_I = 64, d_I = 128 (see the file comment), by
// partials in dk_part (kl_dk_tc_max_items slots of 128 x 128 fp32) with the item offsets in
// offs (batch * ceil(max_seqlen_k / 128) + 1 ints).
int kl_dk_tc_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                    int batch, long long total_q, long long total_k, int max_seqlen_k, long long r0, long long r1,
                    const float* g, long long ld, float* dk_part, int* offs, float* dk_acc, cudaStream_t s) {
  using C = dsa::KlDkCfg;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_dk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  const int tiles = (max_seqlen_k + 127) / 128;
  if (tiles <= 0 || r1 <= r0) return DSA_OK;
  dsa::dk_items_kernel<<<1, 1024, 0, s>>>(cu_q, cu_k, batch, tiles, r0, r1, offs);
  if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  CUtensorMap tk, tq;
  int st = make_tmap_bf16_2d(&tk, k_idx, (uint64_t)total_k, 128, 256, 128, 64, 128);
  if (st != DSA_OK) return st;
  st = make_tmap_bf16_2d(&tq, q_idx, (uint64_t)total_q * 64, 128, 256, 128, 64, 128);
  if (st != DSA_OK) return st;
  dsa::KlDkParams p;
  p.w = static_cast<const uint16_t*>(w);
  p.total_q = total_q;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.row_begin = r0;
  p.row_end = r1;
  p.g = g;
  p.ld = ld;
  p.tiles_per_seq = tiles;
  p.n_pairs = batch * tiles;
  p.offs = offs;
  p.dk_part = dk_part;
  dsa::kl_dk_tc_kernel<<<(unsigned)sm_count(), C::THREADS, C::SMEM_BYTES, s>>>(tk, tq, p);
  if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  // dk_acc += the pairs' slots in item order
  const long long quads = total_k * 32;
  if (quads > 0) {
    dsa::dk_reduce_items_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, s>>>(dk_part, offs, tiles, cu_k, batch,
                                                                               total_k, dk_acc);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

// dw and dq_idx of the row chunk [r0, r1) for H_I = 64, d_I = 128 (row-stationary, above).
int kl_dq_tc_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                    long long total_q, long long total_k, long long r0, long long r1, const float* g, long long ld,
                    void* dq, void* dw, cudaStream_t s) {
  using C = dsa::KlDqCfg;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  CUtensorMap tk, tq;
  int st = make_tmap_bf16_2d(&tk, k_idx, (uint64_t)total_k, 128, 256, 128, 64, 128);
  if (st != DSA_OK) return st;
  st = make_tmap_bf16_2d(&tq, q_idx, (uint64_t)total_q * 64, 128, 256, 128, 64, 128);
  if (st != DSA_OK) return st;
  dsa::KlDqParams p;
  p.q_idx = static_cast<const uint16_t*>(q_idx);
  p.w = static_cast<const uint16_t*>(w);
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.row_begin = r0;
  p.row_end = r1;
  p.g = g;
  p.ld = ld;
  p.dq = static_cast<uint16_t*>(dq);
  p.dw = static_cast<uint16_t*>(dw);
  // an upper bound on the 2-row blocks (each sequence piece rounds up once)
  p.n_blocks = (r1 - r0 + 1) / 2 + batch;
  const long long grid = std::min<long long>(p.n_blocks, (long long)sm_count());
  if (grid <= 0) return DSA_OK;
  p.n_slots = (p.n_blocks + grid - 1) / grid * grid;
  dsa::kl_dq_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tk, tq, p);
  return last_launch_status();
}

}  // namespace dsa_host
