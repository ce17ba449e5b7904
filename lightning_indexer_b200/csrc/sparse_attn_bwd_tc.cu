// Backward of sparse GQA attention as a masked dense pass on tcgen05 tensor cores (sm_100a),
// for d = 128 and 8 query heads per KV head when the selected sets are dense.
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1, sparse-adaptation
// stage (the whole model trains through sparse attention); QbitAI launch article
// (news.chathome.org): varlen DSA training kernels.  Same gradients as the gather kernel
// of sparse_attn_bwd.cu; for token t, head h (KV head g), key s:
//   P = sel(t,s) exp(scale Q.K - lse),  dS = P (dO.V - dO.O)
//   dQ[t,h] = scale sum_s dS K[s,g],  dK[s,g] = scale sum_{t,h} dS Q[t,h],  dV[s,g] = sum_{t,h} P dO[t,h]
// where sel(t,s) is 1 when s is in token t's selected set.  With k selected keys out of at
// most max_seqlen_k visible ones and k >= max_seqlen_k / 8, most causal pairs are selected
// and a dense tile with a selection mask does less work than scattering every selected
// pair's dK and dV rows (1 KiB of fp32 reductions per pair and KV head).
//
// A work item is (128-key tile of one sequence, KV head g); it walks the blocks of 8 tokens
// that see the tile (64 (token, head) rows), keeping dK and dV of the tile in TMEM, so each
// key's dK and dV are written once (no reductions).  Per block, with keys on TMEM lanes:
//   S^T  = K_tile . Q_blk^T,  dP^T = V_tile . dO_blk^T             (N = 64 rows)
//   epilogue  P^T, dS^T -> bf16, 128-byte swizzled rows of 64 (token, head) values
//   dV += P^T . dO_blk,  dK += dS^T . Q_blk                         (B read MN-major)
//   dQ^T[d x rows] = K_tile^T . dS^T                                (A and B read MN-major)
// dQ^T goes to an fp32 accumulator with 16-byte float reductions after a 4 x 4 lane
// transpose (their order can vary between runs; dK and dV are deterministic).  Items are
// taken from a global counter with the KV head slowest, then the sequence, then the key tile
// (long early tiles first), so that the dQ rows the items in flight reduce into (one or two
// sequences of one KV head) stay in L2.  Warps: 0 TMA, 1 MMA issuer and TMEM owner,
// 2-9 epilogue (warp w: keys 32 (w % 4) .., rows 32 ((w - 2) / 4) .. of each block).
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct SABwdTcParams {
  const int* cu_q;
  const int* cu_k;
  int batch, Hq, Hkv;
  int tiles_max;           // ceil(max_seqlen_k / 128)
  long long n_items;       // tiles_max * batch * Hkv
  float scale, scale_log2;
  long long total_q;       // T
  const float2* LD;        // [Hkv, T, 8] (lse in base 2, dO . O) of head 8 g + i
  const uint32_t* mask;    // [tiles_max, T, 4] selection bits: key s is bit s % 32 of word
                           // (s % 128) / 32 of tile s / 128
  float* dQ_acc;           // [T, Hq, 128] fp32, zeroed
  uint16_t* dK;            // [Tk, Hkv, 128] bf16
  uint16_t* dV;
  int* counter;            // item counter, zeroed
};

struct SABwdItem {
  int b, j, g;
  int Lq, Lk, qbase, kbase;
  int blk0, nq;  // first 8-token block that sees the tile, number of blocks
};

__device__ __forceinline__ bool sa_bwd_item(int id, const SABwdTcParams& p, SABwdItem& it) {
  // KV head slowest, then sequence, then key tile (the long early tiles first): the items
  // in flight at a time reduce dQ into the rows of one or two sequences of one KV head,
  // which stay in L2
  it.g = (int)(id / (p.tiles_max * p.batch));
  it.b = (id / p.tiles_max) % p.batch;
  it.j = id % p.tiles_max;
  it.qbase = p.cu_q[it.b];
  it.kbase = p.cu_k[it.b];
  it.Lq = p.cu_q[it.b + 1] - it.qbase;
  it.Lk = p.cu_k[it.b + 1] - it.kbase;
  if (it.j * 128 >= it.Lk) return false;
  // token i sees key s when s < i + Lk - Lq + 1
  const int i_first = max(0, it.j * 128 - (it.Lk - it.Lq));
  if (i_first >= it.Lq) return false;
  it.blk0 = i_first / 8;
  it.nq = (it.Lq + 7) / 8 - it.blk0;
  return true;
}

struct SABwdTcCfg {
  static constexpr int KV_TILE = 128 * 128 * 2;  // 128 keys x 128 dims
  static constexpr int KV_PANEL = 128 * 128;
  static constexpr int QD_TILE = 64 * 128 * 2;   // 8 tokens x 8 heads x 128 dims
  static constexpr int QD_PANEL = 64 * 128;
  static constexpr int LD_BYTES = 8 * 8 * 8;     // float2 of 8 tokens x 8 heads
  static constexpr int MASK_BYTES = 8 * 16;      // 4 words of 8 tokens
  static constexpr int STAGE = 2 * QD_TILE + 1024;  // Q, dO, then LD and mask
  static constexpr int PT_BYTES = 128 * 64 * 2;  // P^T or dS^T: 128 keys x 64 rows
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + KV_TILE;
  static constexpr int QD_STAGES = 3;
  static constexpr int OFF_ST = OFF_V + KV_TILE;                  // QD_STAGES stages
  static constexpr int OFF_P = OFF_ST + QD_STAGES * STAGE;        // P^T, dS^T
  static constexpr int OFF_BAR = OFF_P + 2 * PT_BYTES;
  // kv_full, kv_empty, qd_full[S], qd_empty[S], s_full, s_empty, p_full, p_empty,
  // dq_full[2], dq_empty[2], acc_full, acc_empty, item_full[2], item_empty[2], done
  static constexpr int NUM_BARS = 2 + 2 * QD_STAGES + 2 + 2 + 4 + 2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 32 + 1024;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int TMEM_COLS = 512;  // S^T [0,64) dP^T [64,128) dV [128,256) dK [256,384) dQ^T 2 x 64
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 64);
  static constexpr uint32_t IDESC_KV = idesc_bf16_f32(128, 128) | kIdescBMnMajor;
  static constexpr uint32_t IDESC_Q = idesc_bf16_f32(128, 64) | kIdescAMnMajor | kIdescBMnMajor;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__global__ void __launch_bounds__(SABwdTcCfg::THREADS, 1)
    sa_bwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_do,
                     const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                     const SABwdTcParams p) {
  using C = SABwdTcCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + 1;
  uint64_t* qd_full = bars + 2;                    // [QD_STAGES]
  uint64_t* qd_empty = qd_full + C::QD_STAGES;     // [QD_STAGES]
  uint64_t* s_full = qd_empty + C::QD_STAGES;
  uint64_t* s_empty = s_full + 1;
  uint64_t* p_full = s_full + 2;
  uint64_t* p_empty = s_full + 3;
  uint64_t* dq_full = s_full + 4;                  // [2]
  uint64_t* dq_empty = s_full + 6;                 // [2]
  uint64_t* acc_full = s_full + 8;
  uint64_t* acc_empty = s_full + 9;
  uint64_t* item_full = s_full + 10;               // [2]
  uint64_t* item_empty = s_full + 12;              // [2]
  uint64_t* mma_done = s_full + 14;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  volatile int* item_slot = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 16);  // [2]
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < C::QD_STAGES; ++i) {
      mbar_init(&qd_full[i], 1);
      mbar_init(&qd_empty[i], 1);
    }
    mbar_init(p_full, C::EPI_WARPS);
    mbar_init(p_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&dq_full[i], 1);
      mbar_init(&dq_empty[i], C::EPI_WARPS);
      mbar_init(&item_full[i], 1);
      mbar_init(&item_empty[i], 1 + C::EPI_WARPS);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, C::EPI_WARPS);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, C::EPI_WARPS);
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
    tma_prefetch_desc(&tmap_do);
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // the item of slot number `n` (in publication order), -1 past the last one; called by a
  // whole epilogue warp or by the MMA thread alone (`whole_warp` false)
  auto take_item = [&](long long n, bool whole_warp, bool& ok, int where) -> int {
    const int s = (int)(n & 1);
    if (!(ok = mbar_wait(&item_full[s], (uint32_t)((n >> 1) & 1), abort_flag, where))) return -1;
    const int id = item_slot[s];
    if (whole_warp) __syncwarp();
    if (!whole_warp || lane == 0) mbar_arrive(&item_empty[s]);
    return id;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer (lane 0)
    if (lane == 0) {
      long long n = 0, m = 0, u = 0;  // items published, items loaded, blocks loaded
      bool ok = true;
      while (ok) {
        int id;
        SABwdItem it;
        for (;;) {
          id = atomicAdd(p.counter, 1);
          if (id >= p.n_items) {
            id = -1;
            break;
          }
          if (sa_bwd_item(id, p, it)) break;
        }
        const int s = (int)(n & 1);
        if (!(ok = mbar_wait(&item_empty[s], (uint32_t)((n >> 1) & 1) ^ 1u, abort_flag, 100))) break;
        item_slot[s] = id;
        mbar_arrive(&item_full[s]);  // release: the slot write is visible to the waiters
        ++n;
        if (id < 0) break;
        if (!(ok = mbar_wait(kv_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 101))) break;
        mbar_arrive_expect_tx(kv_full, 2 * C::KV_TILE);
        for (int pn = 0; pn < 2; ++pn) {
          tma_load_3d(smem + C::OFF_K + pn * C::KV_PANEL, &tmap_k, kv_full, pn * 64, it.g, it.kbase + it.j * 128);
          tma_load_3d(smem + C::OFF_V + pn * C::KV_PANEL, &tmap_v, kv_full, pn * 64, it.g, it.kbase + it.j * 128);
        }
        ++m;
        for (int q = 0; q < it.nq; ++q, ++u) {
          const int st = (int)(u % C::QD_STAGES);
          if (!(ok = mbar_wait(&qd_empty[st], (uint32_t)((u / C::QD_STAGES) & 1) ^ 1u, abort_flag, 102))) break;
          const int i0 = (it.blk0 + q) * 8;
          const int ntok = min(8, it.Lq - i0);
          const int t0 = it.qbase + i0;
          uint8_t* sst = smem + C::OFF_ST + st * C::STAGE;
          mbar_arrive_expect_tx(&qd_full[st], 2 * C::QD_TILE + ntok * (64 + 16));
          for (int pn = 0; pn < 2; ++pn) {
            tma_load_3d(sst + pn * C::QD_PANEL, &tmap_q, &qd_full[st], pn * 64, it.g * 8, t0);
            tma_load_3d(sst + C::QD_TILE + pn * C::QD_PANEL, &tmap_do, &qd_full[st], pn * 64, it.g * 8, t0);
          }
          // the block's (lse, D) rows and selection words are contiguous: one copy each
          bulk_g2s(sst + 2 * C::QD_TILE, p.LD + ((size_t)it.g * p.total_q + t0) * 8, ntok * 64, &qd_full[st]);
          bulk_g2s(sst + 2 * C::QD_TILE + C::LD_BYTES, p.mask + ((size_t)it.j * p.total_q + t0) * 4, ntok * 16,
                   &qd_full[st]);
        }
      }
      if (!ok) {
        // let the copies this thread issued land before the CTA exits (bounded)
        const uint64_t t0 = globaltimer_ns();
        for (long long k = max(0LL, u - C::QD_STAGES); k < u; ++k)
          while (!mbar_try_wait(smem_u32(&qd_full[k % C::QD_STAGES]), (uint32_t)((k / C::QD_STAGES) & 1)) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        if (m > 0)
          while (!mbar_try_wait(smem_u32(kv_full), (uint32_t)((m - 1) & 1)) && globaltimer_ns() - t0 < 100000000ull) {
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    long long n = 0, m = 0, u = 0;
    bool ok = true;
    const uint32_t k_base = smem_u32(smem + C::OFF_K);
    const uint32_t v_base = smem_u32(smem + C::OFF_V);
    // S^T and dP^T of block uu (its stage must have landed and S/dP must be free)
    auto mma_s = [&](long long uu) -> bool {
      const int st = (int)(uu % C::QD_STAGES);
      if (!mbar_wait(&qd_full[st], (uint32_t)((uu / C::QD_STAGES) & 1), abort_flag, 103)) return false;
      if (!mbar_wait(s_empty, (uint32_t)(uu & 1) ^ 1u, abort_flag, 104)) return false;
      tc_fence_after();
      const uint32_t q_base = smem_u32(smem + C::OFF_ST + st * C::STAGE);
      const uint32_t do_base = q_base + C::QD_TILE;
#pragma unroll
      for (int pn = 0; pn < 2; ++pn)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const bool acc = (pn | kk) != 0;
          umma_bf16(tmem_base, smem_desc_kmajor(k_base + pn * C::KV_PANEL + kk * 32, 128),
                    smem_desc_kmajor(q_base + pn * C::QD_PANEL + kk * 32, 128), C::IDESC_S, acc);
          umma_bf16(tmem_base + 64, smem_desc_kmajor(v_base + pn * C::KV_PANEL + kk * 32, 128),
                    smem_desc_kmajor(do_base + pn * C::QD_PANEL + kk * 32, 128), C::IDESC_S, acc);
        }
      umma_commit(s_full);
      return true;
    };
    if (lane == 0) {
      while (ok) {
        const int id = take_item(n, false, ok, 105);
        ++n;
        if (!ok || id < 0) break;
        SABwdItem it;
        sa_bwd_item(id, p, it);
        if (!(ok = mbar_wait(kv_full, (uint32_t)(m & 1), abort_flag, 106))) break;
        tc_fence_after();
        if (!(ok = mma_s(u))) break;
        for (int q = 0; q < it.nq && ok; ++q, ++u) {
          if (q + 1 < it.nq && !(ok = mma_s(u + 1))) break;
          const int st = (int)(u % C::QD_STAGES), db = (int)(u & 1);
          if (!(ok = mbar_wait(p_full, (uint32_t)(u & 1), abort_flag, 107))) break;
          if (q == 0 && !(ok = mbar_wait(acc_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 108))) break;
          if (!(ok = mbar_wait(&dq_empty[db], (uint32_t)((u >> 1) & 1) ^ 1u, abort_flag, 109))) break;
          tc_fence_after();
          const uint32_t q_base = smem_u32(smem + C::OFF_ST + st * C::STAGE);
          const uint32_t do_base = q_base + C::QD_TILE;
          const uint32_t pt_base = smem_u32(smem + C::OFF_P);
          const uint32_t ds_base = pt_base + C::PT_BYTES;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 64 rows, 16 per step
            const bool acc = (q | kk) != 0;
            umma_bf16(tmem_base + 128, smem_desc_kmajor(pt_base + kk * 32, 128),
                      smem_desc_mn_sw128(do_base + kk * 16 * 128, C::QD_PANEL), C::IDESC_KV, acc);
            umma_bf16(tmem_base + 256, smem_desc_kmajor(ds_base + kk * 32, 128),
                      smem_desc_mn_sw128(q_base + kk * 16 * 128, C::QD_PANEL), C::IDESC_KV, acc);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // K = 128 keys, 16 per step
            umma_bf16(tmem_base + 384 + db * 64, smem_desc_mn_sw128(k_base + kk * 16 * 128, C::KV_PANEL),
                      smem_desc_mn_sw128(ds_base + kk * 16 * 128, C::PT_BYTES), C::IDESC_Q, kk != 0);
          umma_commit(&dq_full[db]);
          umma_commit(&qd_empty[st]);
          umma_commit(p_empty);
        }
        if (!ok) break;
        umma_commit(acc_full);
        umma_commit(kv_empty);
        ++m;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quarter = warp % 4;
    const int half = (warp - 2) / 4;        // rows 32 half .. (tokens 4 half .. 4 half + 3)
    const int key = quarter * 32 + lane;    // TMEM lane: key of the tile; for dQ^T: dim
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    long long n = 0, m = 0, u = 0;
    bool ok = true;
    // dQ^T of block uu: lanes = dims, columns = this warp's 32 rows -> fp32 reductions
    auto dq_out = [&](long long uu, const SABwdItem& it, int q) -> bool {
      const int st = (int)(uu & 1);
      if (!mbar_wait(&dq_full[st], (uint32_t)((uu >> 1) & 1), abort_flag, 110)) return false;
      tc_fence_after();
      float v[32];
      tmem_ld_x32_sync(tmem_base + lane_off + 384 + st * 64 + half * 32, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dq_empty[st]);
      // 4 x 4 transposes among lanes 4a .. 4a + 3 (two xor-shuffle steps) give lane 4a + b the
      // dims 32 quarter + 4a .. + 3 of row 4 grp + b, so each reduction carries 16 bytes
      const int a = lane >> 2, b = lane & 3;
      const int i0 = (it.blk0 + q) * 8 + 4 * half;
#pragma unroll
      for (int grp = 0; grp < 8; ++grp) {
        float x0 = v[4 * grp], x1 = v[4 * grp + 1], x2 = v[4 * grp + 2], x3 = v[4 * grp + 3];
        {
          const float r0 = __shfl_xor_sync(0xffffffffu, (b & 1) ? x0 : x1, 1);
          const float r1 = __shfl_xor_sync(0xffffffffu, (b & 1) ? x2 : x3, 1);
          if (b & 1) {
            x0 = r0;
            x2 = r1;
          } else {
            x1 = r0;
            x3 = r1;
          }
        }
        {
          const float r0 = __shfl_xor_sync(0xffffffffu, (b & 2) ? x0 : x2, 2);
          const float r1 = __shfl_xor_sync(0xffffffffu, (b & 2) ? x1 : x3, 2);
          if (b & 2) {
            x0 = r0;
            x1 = r1;
          } else {
            x2 = r0;
            x3 = r1;
          }
        }
        const int c = 4 * grp + b;  // column: token 4 half + c / 8, head c % 8
        if (i0 + (c >> 3) < it.Lq)
          red_add_v4(p.dQ_acc + ((size_t)(it.qbase + i0 + (c >> 3)) * p.Hq + it.g * 8 + (c & 7)) * 128 + quarter * 32 +
                         4 * a,
                     x0 * p.scale, x1 * p.scale, x2 * p.scale, x3 * p.scale);
      }
      return true;
    };
    while (ok) {
      const int id = take_item(n, true, ok, 111);
      ++n;
      if (!ok || id < 0) break;
      SABwdItem it;
      sa_bwd_item(id, p, it);
      for (int q = 0; q < it.nq; ++q, ++u) {
        const int st = (int)(u % C::QD_STAGES);
        // this block's lse / D / selection bits arrive with its query tiles
        if (!(ok = mbar_wait(&qd_full[st], (uint32_t)((u / C::QD_STAGES) & 1), abort_flag, 112))) break;
        if (!(ok = mbar_wait(s_full, (uint32_t)(u & 1), abort_flag, 113))) break;
        tc_fence_after();
        float sv[32], dp[32];
        tmem_ld_x32_sync(tmem_base + lane_off + half * 32, sv);
        tmem_ld_x32_sync(tmem_base + lane_off + 64 + half * 32, dp);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_empty);
        const uint8_t* sst = smem + C::OFF_ST + st * C::STAGE;
        const float4* LD4 = reinterpret_cast<const float4*>(sst + 2 * C::QD_TILE) + half * 16;
        const uint32_t* mk = reinterpret_cast<const uint32_t*>(sst + 2 * C::QD_TILE + C::LD_BYTES);
        const int ntok = min(8, it.Lq - (it.blk0 + q) * 8);
        uint32_t pk_p[16], pk_d[16];
#pragma unroll
        for (int tk = 0; tk < 4; ++tk) {
          const int tok = 4 * half + tk;
          const bool sel_any = tok < ntok;
          const uint32_t word = sel_any ? mk[tok * 4 + quarter] : 0u;
          const bool sel = (word >> lane) & 1u;
#pragma unroll
          for (int hp = 0; hp < 4; ++hp) {  // heads 2 hp, 2 hp + 1
            const float4 ld = LD4[tk * 4 + hp];  // (lse2, D) of the two heads
            const int c = tk * 8 + 2 * hp;
            const float p0 = sel ? ex2_ftz(fmaf(sv[c], p.scale_log2, -ld.x)) : 0.f;
            const float p1 = sel ? ex2_ftz(fmaf(sv[c + 1], p.scale_log2, -ld.z)) : 0.f;
            const float d0 = sel ? p0 * (dp[c] - ld.y) : 0.f;
            const float d1 = sel ? p1 * (dp[c + 1] - ld.w) : 0.f;
            __nv_bfloat162 bp = __floats2bfloat162_rn(p0, p1);
            __nv_bfloat162 bd = __floats2bfloat162_rn(d0, d1);
            pk_p[tk * 4 + hp] = *reinterpret_cast<uint32_t*>(&bp);
            pk_d[tk * 4 + hp] = *reinterpret_cast<uint32_t*>(&bd);
          }
        }
        if (!(ok = mbar_wait(p_empty, (uint32_t)(u & 1) ^ 1u, abort_flag, 114))) break;
        // row `key` of P^T and dS^T: 16-byte chunks 4 half .. 4 half + 3 of its 128 bytes
        const uint32_t pt_row = smem_u32(smem + C::OFF_P) + key * 128;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t off = (uint32_t)(((4 * half + c4) ^ (key & 7)) * 16);
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pt_row + off), "r"(pk_p[c4 * 4]),
                       "r"(pk_p[c4 * 4 + 1]), "r"(pk_p[c4 * 4 + 2]), "r"(pk_p[c4 * 4 + 3])
                       : "memory");
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(pt_row + C::PT_BYTES + off),
                       "r"(pk_d[c4 * 4]), "r"(pk_d[c4 * 4 + 1]), "r"(pk_d[c4 * 4 + 2]), "r"(pk_d[c4 * 4 + 3])
                       : "memory");
        }
        fence_proxy_async_shared();  // the tensor core reads P^T and dS^T through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        if (q > 0 && !(ok = dq_out(u - 1, it, q - 1))) break;
      }
      if (!ok) break;
      if (!(ok = dq_out(u - 1, it, it.nq - 1))) break;
      // the tile's dV and dK: one key per lane, this warp's 64 of the 128 dims
      if (!(ok = mbar_wait(acc_full, (uint32_t)(m & 1), abort_flag, 115))) break;
      tc_fence_after();
      const int s = it.j * 128 + key;
      const size_t orow = ((size_t)(it.kbase + s) * p.Hkv + it.g) * 128 + half * 64;
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        uint16_t* dst = (which == 0 ? p.dV : p.dK) + orow;
        const float mul = which == 0 ? 1.f : p.scale;
#pragma unroll 1
        for (int c = 0; c < 64; c += 32) {
          float v[32];
          tmem_ld_x32_sync(tmem_base + lane_off + 128 + which * 128 + half * 64 + c, v);
          if (s < it.Lk) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 o;
              uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(v[e + 2 * f] * mul, v[e + 2 * f + 1] * mul);
                po[f] = *reinterpret_cast<uint32_t*>(&b2);
              }
              *reinterpret_cast<uint4*>(dst + c + e) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      ++m;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// LD[g, t, i] = (lse[t,h] log2(e), dO[t,h] . O[t,h]) for h = 8 g + i; one warp per (t, h),
// d = 128
__global__ void sa_bwd_prep_kernel(const uint16_t* __restrict__ O, const uint16_t* __restrict__ dO,
                                   const float* __restrict__ lse, long long T, int Hq, float2* __restrict__ LD) {
  const long long rows = T * Hq;
  const long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (r >= rows) return;
  const uint2 a = *reinterpret_cast<const uint2*>(O + r * 128 + lane * 4);
  const uint2 b = *reinterpret_cast<const uint2*>(dO + r * 128 + lane * 4);
  float acc = __uint_as_float(a.x << 16) * __uint_as_float(b.x << 16);
  acc = fmaf(__uint_as_float(a.x & 0xFFFF0000u), __uint_as_float(b.x & 0xFFFF0000u), acc);
  acc = fmaf(__uint_as_float(a.y << 16), __uint_as_float(b.y << 16), acc);
  acc = fmaf(__uint_as_float(a.y & 0xFFFF0000u), __uint_as_float(b.y & 0xFFFF0000u), acc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  const long long t = r / Hq;
  const int h = (int)(r % Hq);
  if (lane == 0) LD[((long long)(h / 8) * T + t) * 8 + (h % 8)] = make_float2(lse[r] * 1.4426950408889634f, acc);
}

// selection bits: one thread per (row, slot); -1 slots and positions the row cannot see
// (outside [0, vis)) are skipped, as in the gather kernels
__global__ void sa_bwd_mask_kernel(const int* __restrict__ indices, const int* __restrict__ cu_q,
                                   const int* __restrict__ cu_k, int batch, long long rows, int k, uint32_t* mask,
                                   int tiles) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * k) return;
  const long long row = i / k;
  const int s = indices[i];
  if (s < 0 || s >= tiles * 128) return;
  int lo = 0, hi = batch;
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if ((long long)cu_q[mid] <= row) lo = mid; else hi = mid;
  }
  const int vis = causal_vis((int)(row - cu_q[lo]), cu_q[lo + 1] - cu_q[lo], cu_k[lo + 1] - cu_k[lo]);
  if (s >= vis) return;
  atomicOr(mask + ((long long)(s >> 7) * rows + row) * 4 + ((s >> 5) & 3), 1u << (s & 31));
}

}  // namespace dsa

namespace dsa_host {

int f32_to_bf16_launch(const float* src, void* dst, long long n, cudaStream_t stream);

static size_t r256b(size_t x) { return (x + 255) / 256 * 256; }

// selection words of `indices` (layout of SABwdTcParams::mask) into `mask`, which it clears
// first (total_q * ceil(max_seqlen_k / 128) * 16 bytes)
int sa_bwd_mask_build(const int* indices, const int* cu_q, const int* cu_k, int batch, long long total_q, int k,
                      int max_seqlen_k, uint32_t* mask, cudaStream_t s) {
  const int tiles = (max_seqlen_k + 127) / 128;
  if (const cudaError_t e_ = cudaMemsetAsync(mask, 0, (size_t)total_q * tiles * 16, s); e_ != cudaSuccess)
    return cuda_fail(e_);
  const long long n = total_q * k;
  if (n <= 0) return DSA_OK;
  dsa::sa_bwd_mask_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(indices, cu_q, cu_k, batch, total_q, k, mask,
                                                                        tiles);
  return last_launch_status();
}

bool sa_bwd_tc_eligible(int Hq, int Hkv, int d, int k, int max_seqlen_k) {
  return d == 128 && Hq == 8 * Hkv && max_seqlen_k > 0 && 8LL * k >= (long long)max_seqlen_k;
}

size_t sa_bwd_tc_workspace_bytes(long long total_q, int Hq, int max_seqlen_k) {
  const long long mw = ((long long)max_seqlen_k + 127) / 128 * 4;
  return r256b((size_t)total_q * Hq * 128 * 4) + r256b((size_t)total_q * Hq * 8) + r256b((size_t)total_q * mw * 4) +
         256;
}

int sa_bwd_tc_launch(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* lse,
                     const int* indices, const int* cu_q, const int* cu_k, int batch, long long total_q,
                     long long total_k, int Hq, int Hkv, int k, int max_seqlen_k, float scale, void* dQ, void* dK,
                     void* dV, void* ws, cudaStream_t s) {
  using C = dsa::SABwdTcCfg;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sa_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  const int mw = (max_seqlen_k + 127) / 128 * 4;
  uint8_t* w = static_cast<uint8_t*>(ws);
  float* dq_acc = reinterpret_cast<float*>(w);
  w += r256b((size_t)total_q * Hq * 128 * 4);
  float2* LD = reinterpret_cast<float2*>(w);
  w += r256b((size_t)total_q * Hq * 8);
  uint32_t* mask = reinterpret_cast<uint32_t*>(w);
  w += r256b((size_t)total_q * mw * 4);
  int* counter = reinterpret_cast<int*>(w);
  // dQ accumulator, selection bits and the item counter start at zero
  if (const cudaError_t e_ = cudaMemsetAsync(ws, 0, sa_bwd_tc_workspace_bytes(total_q, Hq, max_seqlen_k), s);
      e_ != cudaSuccess)
    return cuda_fail(e_);
  // keys no block reaches (sequences without queries) keep zero gradients
  if (const cudaError_t e_ = cudaMemsetAsync(dK, 0, (size_t)total_k * Hkv * 128 * 2, s); e_ != cudaSuccess)
    return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemsetAsync(dV, 0, (size_t)total_k * Hkv * 128 * 2, s); e_ != cudaSuccess)
    return cuda_fail(e_);
  if (total_q > 0) {
    const long long rows = total_q * Hq;
    dsa::sa_bwd_prep_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(
        static_cast<const uint16_t*>(O), static_cast<const uint16_t*>(dO), lse, total_q, Hq, LD);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
    const long long n = total_q * k;
    dsa::sa_bwd_mask_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(indices, cu_q, cu_k, batch, total_q, k, mask,
                                                                        mw / 4);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  }
  CUtensorMap tq, tdo, tk, tv;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)std::max<long long>(total_q, 1)};
    const uint64_t strides[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 8, 8};
    if (const int st = make_tmap_bf16_3d(&tq, Q, dims, strides, box); st != DSA_OK) return st;
    if (const int st = make_tmap_bf16_3d(&tdo, dO, dims, strides, box); st != DSA_OK) return st;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)std::max<long long>(total_k, 1)};
    const uint64_t strides[2] = {256, (uint64_t)Hkv * 256};
    const uint32_t box[3] = {64, 1, 128};
    if (const int st = make_tmap_bf16_3d(&tk, K, dims, strides, box); st != DSA_OK) return st;
    if (const int st = make_tmap_bf16_3d(&tv, V, dims, strides, box); st != DSA_OK) return st;
  }
  dsa::SABwdTcParams p;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.tiles_max = (max_seqlen_k + 127) / 128;
  p.n_items = (long long)p.tiles_max * batch * Hkv;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.total_q = total_q;
  p.LD = LD;
  p.mask = mask;
  p.dQ_acc = dq_acc;
  p.dK = static_cast<uint16_t*>(dK);
  p.dV = static_cast<uint16_t*>(dV);
  p.counter = counter;
  const long long grid = std::min<long long>(p.n_items, (long long)sm_count());
  if (grid > 0 && total_q > 0) {
    dsa::sa_bwd_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tdo, tk, tv, p);
    if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  }
  return f32_to_bf16_launch(dq_acc, dQ, total_q * Hq * 128, s);
}

}  // namespace dsa_host
