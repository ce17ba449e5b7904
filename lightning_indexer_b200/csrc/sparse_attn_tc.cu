// Sparse GQA attention (prefill) as a masked dense pass on tcgen05 tensor cores (sm_100a),
// for d = 128 and 8 query heads per KV head when the selected sets are dense.
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1 (each token attends to
// its top-k selected positions; GQA adaptation).  For token t, head h (KV head g):
//   O[t,h] = sum_{s selected} softmax_s(scale Q[t,h].K[s,g]) V[s,g],  lse[t,h] = log sum exp
// With k selected keys out of at most max_seqlen_k visible ones and k >= max_seqlen_k / 8,
// most causal pairs are selected, and dense 128 x 128 tiles with a selection mask do less
// work than gathering every selected key's K and V rows per (token, KV head).
//
// Two passes over the same work items, (16 query rows of one sequence, KV head g): the
// first is the dense-LSE kernel of kl_dense_tc.cu run with the selection mask (it writes
// lse and the row maxima m); the second, below, recomputes S = Q_blk . K_tile^T (M = 16
// tokens x 8 heads on TMEM lanes, N = 128 keys), turns it into P = sel 2^(S scale log2(e) - m)
// (in [0, 1], the largest exactly 1; written to tensor memory as two bf16 parts, hi + lo),
// accumulates O += P_hi . V_tile + P_lo . V_tile in TMEM with P read from tensor memory and
// V from shared memory (MN-major), and divides by the row sum 2^(lse - m) in fp32 at the end.
// Knowing m first removes the running rescale of O.  Warps: 0 TMA, 1 MMA issuer and TMEM
// owner, 4-11 epilogue (two per TMEM lane quarter, one per 64-key half of each tile), and six
// gather warps for the union form below.
//
// Adjacent-query reuse (report summary section 8: neighbouring queries select largely the
// same positions; the pages deduplicate the sets of adjacent queries and mask inside the
// attention kernel with a mask laid out like the MMA's accumulator): the same two passes in
// their union form, where a 16-row block visits the 128-position chunks of the sorted union
// of its rows' selected sets, copied row by row by two gather warps with 16-byte cp.async
// into the swizzled tiles (each key loaded once for the 16 rows x 8 heads of the block), and
// the per-(row, union slot) selection bits mask S.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct SAFwdTcParams {
  KlLseParams items;      // work items and selection words (shared with the LSE pass)
  const uint16_t* K;      // union form: K and V [Tk, Hkv, 128] bf16, read by the gather warps
  const uint16_t* V;
  const float* lse;       // [T, Hq] natural log (first pass)
  const float* mx;        // [T, Hq] row maxima of the scaled logits, base 2 (first pass)
  uint16_t* O;            // [T, Hq, 128] bf16
};

struct SAFwdTcCfg {
  static constexpr int TILE_BYTES = 128 * 128 * 2;
  static constexpr int PANEL_BYTES = 128 * 128;
  // K tiles are free after their S MMA, V tiles only after P.V: separate rings (P lives in
  // tensor memory, so shared memory holds only Q and the rings)
  static constexpr int K_STAGES = 3, V_STAGES = 3;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + K_STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_V + V_STAGES * TILE_BYTES;
  // q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full[2], s_empty[2],
  // p_full, p_empty, o_full, o_empty, done
  static constexpr int NUM_BARS = 2 + 2 * K_STAGES + 2 * V_STAGES + 4 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // Warps: 0 TMA, 1 MMA and TMEM, 2-3 K gather (warpgroup 0); 4-11 epilogue (warpgroups 1-2);
  // 12 K gather, 13-15 V gather (warpgroup 3).  The gather warps copy the union form's K and
  // V chunks with cp.async and idle otherwise.  Registers after the reallocation: 80 for
  // warpgroup 0, 176 for the epilogue, 64 for warpgroup 3 (128 x 80 + 256 x 176 + 128 x 64 =
  // 63488 of the 65536 that 512 threads at 128 registers hold).
  static constexpr int EPI_WARPS = 8;
  static constexpr int GATHER_K = 3, GATHER_V = 3;
  static constexpr int THREADS = 512;
  static constexpr int REG_WG0 = 80, REG_EPI = 176, REG_WG3 = 64;
  // S [0,128) [128,256), O [256,384), P_hi [384,448), P_lo [448,512) (two bf16 per column)
  static constexpr int TMEM_COLS = 512;
  static constexpr int TM_O = 256, TM_PHI = 384, TM_PLO = 448;
  static constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128);
  static constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 128) | kIdescBMnMajor;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(SAFwdTcCfg::THREADS, 1)
    sa_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const SAFwdTcParams p) {
  using C = SAFwdTcCfg;
  const KlLseParams& ip = p.items;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;                    // [K_STAGES]
  uint64_t* k_empty = k_full + C::K_STAGES;       // [K_STAGES]
  uint64_t* v_full = k_empty + C::K_STAGES;       // [V_STAGES]
  uint64_t* v_empty = v_full + C::V_STAGES;       // [V_STAGES]
  uint64_t* s_full = v_empty + C::V_STAGES;       // [2]
  uint64_t* s_empty = s_full + 2;                 // [2]
  uint64_t* p_full = s_full + 4;
  uint64_t* p_empty = s_full + 5;
  uint64_t* o_full = s_full + 6;
  uint64_t* o_empty = s_full + 7;
  uint64_t* mma_done = s_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < C::K_STAGES; ++i) {
      mbar_init(&k_full[i], ip.ukeys ? C::GATHER_K * 32 : 1);  // TMA, or the K gather lanes
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::V_STAGES; ++i) {
      mbar_init(&v_full[i], ip.ukeys ? C::GATHER_V * 32 : 1);
      mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], C::EPI_WARPS);
    }
    mbar_init(p_full, C::EPI_WARPS);
    mbar_init(p_empty, 1);
    mbar_init(o_full, 1);
    mbar_init(o_empty, C::EPI_WARPS);
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
    tma_prefetch_desc(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int G = ip.Hq / ip.Hkv;  // 8
  const long long n_items = kl_item_count(ip);

  // ------------------------------------------------------------ gather warps (union form),
  // in warpgroups 0 and 3: warps 2, 3, 12 copy the K chunks, 13-15 the V chunks, so that a K
  // copy never waits behind a V stage (freed only after its P.V)
  auto gather_role = [&]() {
    if (ip.ukeys) {
      const bool is_v = warp >= 13;
      const int wg = is_v ? warp - 13 : (warp == 12 ? 2 : warp - 2);
      const int nw = is_v ? C::GATHER_V : C::GATHER_K;
      const int stages = is_v ? C::V_STAGES : C::K_STAGES;
      uint64_t* full = is_v ? v_full : k_full;
      uint64_t* empty = is_v ? v_empty : k_empty;
      uint8_t* ring = smem + (is_v ? C::OFF_V : C::OFF_K);
      const uint16_t* src = is_v ? p.V : p.K;
      long long n = 0;
      bool ok = true;
      for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        KlLseItem it;
        if (!kl_lse_item(item, ip, it) || it.ntiles == 0) continue;
        const int* keys = ip.ukeys + it.blk * ip.ucap;
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int st = (int)(n % stages);
          if (lane == 0) ok = mbar_wait(&empty[st], (uint32_t)((n / stages) & 1) ^ 1u, abort_flag, is_v ? 133 : 132);
          if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
          union_copy_tile(ring + st * C::TILE_BYTES, C::PANEL_BYTES, src, keys + j * 128, it.kbase, ip.Hkv, it.g, nw,
                          wg, lane, &full[st]);
        }
      }
      cp_async_wait<0>();  // nothing of this thread's in flight when the CTA leaves
    }
  };
  if (warp < 4) {
    setmaxnreg_dec<C::REG_WG0>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer (the query
      // block of each item; the K and V tiles too, except in the union form)
      long long m = 0, n = 0;    // items with key tiles, key tiles
      long long nk = 0, nv = 0;  // K and V tile copies issued (they differ after an abort)
      bool ok = true;
      if (lane == 0) {
        for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
          KlLseItem it;
          if (!kl_lse_item(item, ip, it) || it.ntiles == 0) continue;
          if (!(ok = mbar_wait(q_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 120))) break;
          mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(smem + C::OFF_Q + pn * C::PANEL_BYTES, &tmap_q, q_full, pn * 64, it.g * G, (int)it.t0);
          ++m;
          if (ip.ukeys) continue;  // the gather warps copy the union chunks
          for (int j = 0; j < it.ntiles; ++j, ++n) {
            const int ks = (int)(n % C::K_STAGES), vs = (int)(n % C::V_STAGES);
            uint8_t* kdst = smem + C::OFF_K + ks * C::TILE_BYTES;
            uint8_t* vdst = smem + C::OFF_V + vs * C::TILE_BYTES;
            if (!(ok = mbar_wait(&k_empty[ks], (uint32_t)((n / C::K_STAGES) & 1) ^ 1u, abort_flag, 121))) break;
            mbar_arrive_expect_tx(&k_full[ks], C::TILE_BYTES);
            for (int pn = 0; pn < 2; ++pn)
              tma_load_3d(kdst + pn * C::PANEL_BYTES, &tmap_k, &k_full[ks], pn * 64, it.g, it.kbase + j * 128);
            ++nk;
            if (!(ok = mbar_wait(&v_empty[vs], (uint32_t)((n / C::V_STAGES) & 1) ^ 1u, abort_flag, 130))) break;
            mbar_arrive_expect_tx(&v_full[vs], C::TILE_BYTES);
            for (int pn = 0; pn < 2; ++pn)
              tma_load_3d(vdst + pn * C::PANEL_BYTES, &tmap_v, &v_full[vs], pn * 64, it.g, it.kbase + j * 128);
            ++nv;
          }
        }
        if (!ok) {
          // let the copies this thread issued land before the CTA exits (bounded; each ring
          // waits only for copies it really issued, each with its own time budget)
          uint64_t t0 = globaltimer_ns();
          for (long long k = max(0LL, nk - C::K_STAGES); k < nk; ++k)
            while (!mbar_try_wait(smem_u32(&k_full[k % C::K_STAGES]), (uint32_t)((k / C::K_STAGES) & 1)) &&
                   globaltimer_ns() - t0 < 100000000ull) {
            }
          t0 = globaltimer_ns();
          for (long long k = max(0LL, nv - C::V_STAGES); k < nv; ++k)
            while (!mbar_try_wait(smem_u32(&v_full[k % C::V_STAGES]), (uint32_t)((k / C::V_STAGES) & 1)) &&
                   globaltimer_ns() - t0 < 100000000ull) {
            }
          t0 = globaltimer_ns();
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
        const uint32_t q_base = smem_u32(smem + C::OFF_Q);
        // S of key tile number nn (its stage landed, its TMEM buffer free)
        auto mma_s = [&](long long nn) -> bool {
          const int ks = (int)(nn % C::K_STAGES), sb = (int)(nn & 1);
          if (!mbar_wait(&k_full[ks], (uint32_t)((nn / C::K_STAGES) & 1), abort_flag, 122)) return false;
          if (!mbar_wait(&s_empty[sb], (uint32_t)((nn >> 1) & 1) ^ 1u, abort_flag, 123)) return false;
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + C::OFF_K + ks * C::TILE_BYTES);
  #pragma unroll
          for (int pn = 0; pn < 2; ++pn)
  #pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(tmem_base + sb * 128, smem_desc_kmajor(q_base + pn * C::PANEL_BYTES + kk * 32, 128),
                        smem_desc_kmajor(k_base + pn * C::PANEL_BYTES + kk * 32, 128), C::IDESC_S, (pn | kk) != 0);
          umma_commit(&s_full[sb]);
          umma_commit(&k_empty[ks]);
          return true;
        };
        for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
          KlLseItem it;
          if (!kl_lse_item(item, ip, it) || it.ntiles == 0) continue;
          if (!(ok = mbar_wait(q_full, (uint32_t)(m & 1), abort_flag, 124))) break;
          tc_fence_after();
          if (!(ok = mma_s(n))) break;
          for (int j = 0; j < it.ntiles && ok; ++j) {
            const long long nn = n + j;
            if (j + 1 < it.ntiles && !(ok = mma_s(nn + 1))) break;
            if (j + 1 == it.ntiles) umma_commit(q_empty);  // the query block is free after the S MMAs
            if (!(ok = mbar_wait(p_full, (uint32_t)(nn & 1), abort_flag, 125))) break;
            if (j == 0 && !(ok = mbar_wait(o_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 126))) break;
            tc_fence_after();
            const int vs = (int)(nn % C::V_STAGES);
            if (!(ok = mbar_wait(&v_full[vs], (uint32_t)((nn / C::V_STAGES) & 1), abort_flag, 131))) break;
            tc_fence_after();
            const uint32_t v_base = smem_u32(smem + C::OFF_V + vs * C::TILE_BYTES);
#pragma unroll
            for (int part = 0; part < 2; ++part)  // P = P_hi + P_lo, both bf16, from tensor memory
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)  // K = 128 keys, 16 per step (8 columns of P)
                umma_bf16_ta(tmem_base + C::TM_O, tmem_base + (part ? C::TM_PLO : C::TM_PHI) + kk * 8,
                             smem_desc_mn_sw128(v_base + kk * 16 * 128, C::PANEL_BYTES), C::IDESC_O,
                             (j | part | kk) != 0);
            umma_commit(&v_empty[vs]);
            umma_commit(p_empty);
          }
          if (!ok) break;
          umma_commit(o_full);
          n += it.ntiles;
          ++m;
        }
        umma_commit(mma_done);
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
        }
      }
    } else {
      gather_role();
    }
  } else if (warp < 4 + C::EPI_WARPS) {
    setmaxnreg_inc<C::REG_EPI>();
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quarter = warp % 4;
    const int half = (warp - 4) / 4;    // keys 64 half .. 64 half + 63 of each tile; O dims likewise
    const int r = quarter * 32 + lane;  // (token, head) of this lane: token r / 8, head r % 8
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    long long m = 0, n = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      KlLseItem it;
      if (!kl_lse_item(item, ip, it)) continue;
      const int u = r / 8;
      const bool valid = u < it.ntok;
      const long long row = (it.t0 + (valid ? u : 0)) * ip.Hq + it.g * G + (r % 8);
      uint16_t* orow = p.O + row * 128 + half * 64;
      if (it.ntiles == 0) {  // no visible key: O = 0 (the first pass wrote lse = -inf)
        if (valid)
#pragma unroll
          for (int e = 0; e < 64; e += 8) *reinterpret_cast<uint4*>(orow + e) = make_uint4(0u, 0u, 0u, 0u);
        continue;
      }
      // P relative to the row maximum; O / sum at the end (rows without a key: O = 0)
      const float lse2 = valid ? p.lse[row] * 1.4426950408889634f : -INFINITY;
      const float nl = valid ? -p.mx[row] : 0.f;
      const float o_scale = lse2 > -INFINITY ? ex2_ftz(-nl - lse2) : 0.f;
      long long mstride;
      const uint32_t* mrow = kl_mask_row(ip, it, valid ? u : 0, mstride) + 2 * half;
      MaskWords mw(valid ? mrow : nullptr, mstride, it.ntiles, 0u);
      for (int j = 0; j < it.ntiles; ++j, ++n) {
        const int sb = (int)(n & 1);
        const uint2 wj = mw.next(j);
        const uint32_t w0 = wj.x, w1 = wj.y;
        if (!(ok = mbar_wait(&s_full[sb], (uint32_t)((n >> 1) & 1), abort_flag, 127))) break;
        tc_fence_after();
        float x[64];
        tmem_ld_x32_sync(tmem_base + lane_off + sb * 128 + half * 64, x);
        tmem_ld_x32_sync(tmem_base + lane_off + sb * 128 + half * 64 + 32, x + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        // P in two bf16 parts, hi = bf16(P) and lo = bf16(P - hi): their sum carries P to about
        // 2^-17 relative, so the weights entering P.V are not the 2^-9 relative rounding of a
        // single bf16 (which, on rows with few keys and values of magnitude 2-4, would add
        // up to the output's own rounding and exceed 1e-2)
        uint32_t pk[32], pl[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const uint32_t w = c < 32 ? w0 : w1;
          const float p0 = ((w >> (c & 31)) & 1u) ? ex2_ftz(fmaf(x[c], ip.scale_log2, nl)) : 0.f;
          const float p1 = ((w >> ((c + 1) & 31)) & 1u) ? ex2_ftz(fmaf(x[c + 1], ip.scale_log2, nl)) : 0.f;
          const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
          const __nv_bfloat162 lo = __floats2bfloat162_rn(p0 - __low2float(hi), p1 - __high2float(hi));
          pk[c / 2] = *reinterpret_cast<const uint32_t*>(&hi);
          pl[c / 2] = *reinterpret_cast<const uint32_t*>(&lo);
        }
        if (!(ok = mbar_wait(p_empty, (uint32_t)(n & 1) ^ 1u, abort_flag, 128))) break;
        tc_fence_after();
        // this row's 64 keys of P: columns 32 half .. 32 half + 31 of the P_hi and P_lo regions
        tmem_st_x32_sync(tmem_base + lane_off + C::TM_PHI + half * 32, pk);
        tmem_st_x32_sync(tmem_base + lane_off + C::TM_PLO + half * 32, pl);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(o_full, (uint32_t)(m & 1), abort_flag, 129))) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld_x32_sync(tmem_base + lane_off + C::TM_O + half * 64 + c, v);
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 o;
            uint32_t* po = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v[e + 2 * f] * o_scale, v[e + 2 * f + 1] * o_scale);
              po[f] = *reinterpret_cast<uint32_t*>(&b2);
            }
            *reinterpret_cast<uint4*>(orow + c + e) = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_empty);
      ++m;
    }
  } else {
    setmaxnreg_dec<C::REG_WG3>();
    gather_role();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------- union plans
// Per block of 16 consecutive query rows (the work items of the two passes): the sorted union
// of the rows' selected positions, through a bitmap of the sequence's positions.  A block
// whose union has at most `ucap` positions takes the union form; the others' rows go to the
// gather kernel.
struct SAUnionPlanParams {
  const int* indices;  // [T, k] (k a multiple of 16)
  int k;
  const int* cu_q;
  const int* cu_k;
  int batch;
  int ucap;              // union positions per block, a multiple of 128
  float max_union_frac;  // the union form only where union <= this x the block's selections
  int* ukeys;            // [n_blocks, ucap]: ascending positions, the last chunk padded with 0
  int* ucount;           // [n_blocks]: union size (also where it exceeds ucap)
  uint32_t* umask;       // [n_blocks, ucap / 128, 16, 4]: bit slot % 32 of word slot / 32 % 4
  uint8_t* blk_use;      // [n_blocks]
  uint8_t* row_tc;       // [T]: 1 for rows of union-form blocks
  int* blk_list;         // the union-form blocks, in no particular order
  int* n_used;           // their number (zeroed before the launch)
};

constexpr int SA_PLAN_T = 256;

// Dynamic shared memory: the position bitmap and its word prefix counts (words each), then
// the block's selection words (ucap / 128 * 64).
__global__ void __launch_bounds__(SA_PLAN_T) sa_union_plan_kernel(const SAUnionPlanParams p, int words) {
  extern __shared__ __align__(16) uint32_t plan_smem[];
  uint32_t* bits = plan_smem;
  uint32_t* pre = plan_smem + words;
  uint32_t* msk = plan_smem + 2 * words;
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t total, nsel_sh;
  long long r = blockIdx.x;
  const long long blk = r;
  int b = 0;
  for (; b < p.batch; ++b) {
    const long long nb = (p.cu_q[b + 1] - p.cu_q[b] + 15) / 16;
    if (r < nb) break;
    r -= nb;
  }
  if (b == p.batch) return;  // past the last block (the bound rounds up per sequence)
  const int Lq = p.cu_q[b + 1] - p.cu_q[b], Lk = p.cu_k[b + 1] - p.cu_k[b];
  const int i0 = (int)(r * 16), ntok = min(16, Lq - i0);
  const long long t0 = p.cu_q[b] + i0;
  const int W = (Lk + 31) / 32;
  const int mwords = p.ucap / 128 * 64;
  for (int w = threadIdx.x; w < W; w += SA_PLAN_T) bits[w] = 0u;
  if (threadIdx.x == 0) nsel_sh = 0u;
  __syncthreads();
  // the rows' valid entries into the bitmap, four indices per load (k is a multiple of 16)
  const int4* idx4 = reinterpret_cast<const int4*>(p.indices + t0 * p.k);
  const int n4 = ntok * p.k / 4;
  uint32_t nsel = 0;
#pragma unroll 4
  for (int e = threadIdx.x; e < n4; e += SA_PLAN_T) {
    const int4 v = __ldg(idx4 + e);
    const int vis = causal_vis(i0 + (4 * e) / p.k, Lq, Lk);
    const int sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (sv[q] >= 0 && sv[q] < vis) {
        atomicOr(&bits[sv[q] >> 5], 1u << (sv[q] & 31));
        ++nsel;
      }
  }
  nsel = __reduce_add_sync(0xffffffffu, nsel);
  if ((threadIdx.x & 31) == 0) atomicAdd(&nsel_sh, nsel);
  __syncthreads();
  // a contiguous run of words per thread; the block scan numbers the union in position order
  const int wpt = (W + SA_PLAN_T - 1) / SA_PLAN_T;
  const int w0 = min(W, (int)threadIdx.x * wpt), w1 = min(W, w0 + wpt);
  uint32_t mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bits[w]);
  uint32_t run = block_excl_scan<SA_PLAN_T>(mine, warp_sums, &total);
  const uint32_t u_n = total;
  // the tensor-core form pays where the block's union is small against its selections (its
  // cost grows with union chunks, the gather kernel's with selections)
  const bool use = u_n <= (uint32_t)p.ucap && (float)u_n <= p.max_union_frac * (float)nsel_sh;
  if (threadIdx.x == 0) {
    p.ucount[blk] = (int)u_n;
    p.blk_use[blk] = use ? 1 : 0;
    if (use) p.blk_list[atomicAdd(p.n_used, 1)] = (int)blk;
  }
  if (threadIdx.x < ntok) p.row_tc[t0 + threadIdx.x] = use ? 1 : 0;
  if (!use) return;  // block-uniform
  for (int w = threadIdx.x; w < mwords; w += SA_PLAN_T) msk[w] = 0u;
  int* keys = p.ukeys + blk * p.ucap;
  for (int w = w0; w < w1; ++w) {
    pre[w] = run;
    uint32_t x = bits[w];
    while (x) {
      keys[run++] = w * 32 + (__ffs(x) - 1);
      x &= x - 1u;
    }
  }
  const uint32_t u_pad = (u_n + 127) / 128 * 128;
  for (uint32_t j = u_n + threadIdx.x; j < u_pad; j += SA_PLAN_T) keys[j] = 0;
  __syncthreads();  // pre[] complete for every word, msk[] cleared
#pragma unroll 4
  for (int e = threadIdx.x; e < n4; e += SA_PLAN_T) {
    const int4 v = __ldg(idx4 + e);
    const int u = (4 * e) / p.k;
    const int vis = causal_vis(i0 + u, Lq, Lk);
    const int sv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int s = sv[q];
      if (s >= 0 && s < vis) {
        const uint32_t slot = pre[s >> 5] + __popc(bits[s >> 5] & ((1u << (s & 31)) - 1u));
        atomicOr(&msk[((slot >> 7) * 16 + u) * 4 + ((slot >> 5) & 3)], 1u << (slot & 31));
      }
    }
  }
  __syncthreads();
  uint32_t* out = p.umask + blk * (long long)mwords;
  for (uint32_t w = threadIdx.x; w < u_pad / 128 * 64; w += SA_PLAN_T) out[w] = msk[w];
}

}  // namespace dsa

namespace dsa_host {

int kl_lse_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                     long long Tk, int Hq, int Hkv, int max_seqlen_q, float scale_log2, float* lse_out,
                     cudaStream_t s, const uint32_t* mask, float out_scale, float* max_out,
                     const KlUnion* un);

// One-time set-up of the O-pass kernel on the current device: its shared memory, and a check
// that the register reallocation fits what a launch holds (else the increase would wait
// for registers that never come).
static int sa_fwd_tc_setup() {
  using C = dsa::SAFwdTcCfg;
  static DeviceFlag done;
  if (done) return DSA_OK;
  if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  C::SMEM_BYTES);
      e_ != cudaSuccess)
    return cuda_fail(e_);
  cudaFuncAttributes fa;
  if (const cudaError_t e_ = cudaFuncGetAttributes(&fa, dsa::sa_fwd_tc_kernel); e_ != cudaSuccess) return cuda_fail(e_);
  if ((long long)fa.numRegs * C::THREADS < 128LL * (C::REG_WG0 + C::REG_WG3) + 256LL * C::REG_EPI)
    return DSA_ERR_UNSUPPORTED;
  done = true;
  return DSA_OK;
}

bool sa_fwd_tc_eligible(int Hq, int Hkv, int d, int k, int max_seqlen_k) {
  return d == 128 && Hq == 8 * Hkv && max_seqlen_k > 0 && 8LL * k >= (long long)max_seqlen_k;
}

// scratch of the two passes: selection words (layout of KlLseParams::mask), then the row
// maxima [T, Hq] fp32
static size_t sa_fwd_tc_mask_only(long long total_q, int max_seqlen_k) {
  return ((size_t)total_q * (size_t)((max_seqlen_k + 127) / 128) * 16 + 255) / 256 * 256;
}
size_t sa_fwd_tc_scratch_bytes(long long total_q, int Hq, int max_seqlen_k) {
  return sa_fwd_tc_mask_only(total_q, max_seqlen_k) + (size_t)total_q * Hq * 4;
}

int sa_bwd_mask_build(const int* indices, const int* cu_q, const int* cu_k, int batch, long long total_q, int k,
                      int max_seqlen_k, uint32_t* mask, cudaStream_t s);

// O and lse of the selected sets in `indices` by the two masked dense passes; `mask_ws`
// holds sa_fwd_tc_scratch_bytes.
int sa_fwd_tc_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                     const int* cu_k, int batch, long long total_q, long long total_k, int Hq, int Hkv, int k,
                     int max_seqlen_k, float scale, void* O, float* lse, void* mask_ws, cudaStream_t s) {
  using C = dsa::SAFwdTcCfg;
  if (const int st = sa_fwd_tc_setup(); st != DSA_OK) return st;
  if (total_q <= 0) return DSA_OK;
  uint32_t* mask = static_cast<uint32_t*>(mask_ws);
  float* mx = reinterpret_cast<float*>(static_cast<uint8_t*>(mask_ws) + sa_fwd_tc_mask_only(total_q, max_seqlen_k));
  int st = sa_bwd_mask_build(indices, cu_q, cu_k, batch, total_q, k, max_seqlen_k, mask, s);
  if (st != DSA_OK) return st;
  const float scale_log2 = scale * 1.4426950408889634f;
  st = kl_lse_tc_launch(Q, K, cu_q, cu_k, batch, total_q, total_k, Hq, Hkv, 0, scale_log2, lse, s, mask,
                        0.69314718055994531f, mx, nullptr);
  if (st != DSA_OK) return st;
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)total_q};
    const uint64_t strides[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 8, 16};
    if (const int e = make_tmap_bf16_3d(&tq, Q, dims, strides, box); e != DSA_OK) return e;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)std::max<long long>(total_k, 1)};
    const uint64_t strides[2] = {256, (uint64_t)Hkv * 256};
    const uint32_t box[3] = {64, 1, 128};
    if (const int e = make_tmap_bf16_3d(&tk, K, dims, strides, box); e != DSA_OK) return e;
    if (const int e = make_tmap_bf16_3d(&tv, V, dims, strides, box); e != DSA_OK) return e;
  }
  dsa::SAFwdTcParams p{};
  p.items.cu_q = cu_q;
  p.items.cu_k = cu_k;
  p.items.batch = batch;
  p.items.Hq = Hq;
  p.items.Hkv = Hkv;
  p.items.scale_log2 = scale_log2;
  p.items.lse_out = lse;
  p.items.out_scale = 1.f;
  p.items.n_blocks = (total_q + 15) / 16 + batch;
  p.items.n_items = p.items.n_blocks * Hkv;
  p.items.mask = mask;
  p.items.total_q = total_q;
  p.items.max_out = nullptr;
  p.lse = lse;
  p.mx = mx;
  p.O = static_cast<uint16_t*>(O);
  const long long grid = std::min<long long>(p.items.n_items, (long long)sm_count());
  dsa::sa_fwd_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, tv, p);
  return last_launch_status();
}

// ---------------------------------------------------------------------------- union path
// Scratch of sa_block_reuse_launch: the row maxima, the per-block unions, their sizes,
// selection words and flags, and the per-row flags.
struct SAUnionWs {
  float* mx;
  int* ukeys;
  int* ucount;
  uint32_t* umask;
  uint8_t* blk_use;
  uint8_t* row_tc;
  int* blk_list;
  int* n_used;
  int ucap;
  size_t total;
};

// A block takes the union form where its union holds at most this fraction of its valid
// selections: on B200 the two tensor-core passes cost about 4.7 us per 128-position chunk
// and KV head on one SM, the gather kernel about 6.5 ns per selected (row, position) pair
// and KV head, so the form pays up to a union of about 0.18 x the selections.
constexpr float kUnionMaxFrac = 0.16f;

// Union positions per block: at most `max_chunks` chunks of 128, and no more than the
// longest sequence holds.
static int sa_union_cap(int max_seqlen_k, int max_chunks) {
  return std::max(1, std::min(max_chunks, (max_seqlen_k + 127) / 128)) * 128;
}

static SAUnionWs sa_union_layout(void* base, long long total_q, int Hq, int batch, int max_seqlen_k, int max_chunks) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  SAUnionWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  const long long n_blocks = (total_q + 15) / 16 + batch;
  w.ucap = sa_union_cap(max_seqlen_k, max_chunks);
  w.mx = reinterpret_cast<float*>(p + off);
  off += up((size_t)total_q * Hq * 4);
  w.ukeys = reinterpret_cast<int*>(p + off);
  off += up((size_t)n_blocks * w.ucap * 4);
  w.ucount = reinterpret_cast<int*>(p + off);
  off += up((size_t)n_blocks * 4);
  w.umask = reinterpret_cast<uint32_t*>(p + off);
  off += up((size_t)n_blocks * (w.ucap / 128) * 256);
  w.blk_use = p + off;
  off += up((size_t)n_blocks);
  w.row_tc = p + off;
  off += up((size_t)total_q);
  w.blk_list = reinterpret_cast<int*>(p + off);
  off += up((size_t)n_blocks * 4);
  w.n_used = reinterpret_cast<int*>(p + off);
  off += 256;
  w.total = off;
  return w;
}

size_t sa_block_reuse_scratch_bytes(long long total_q, int Hq, int batch, int max_seqlen_k, int max_chunks) {
  return sa_union_layout(nullptr, total_q, Hq, batch, max_seqlen_k, max_chunks).total;
}

// The union plan holds a bitmap of a sequence's positions and its prefix counts in shared
// memory: 2 x 32 KiB at 262144 positions.
bool sa_block_reuse_eligible(int Hq, int Hkv, int d, int max_seqlen_k) {
  return d == 128 && Hq == 8 * Hkv && max_seqlen_k > 0 && max_seqlen_k <= 262144;
}

int sparse_attn_prefill_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                               const int* cu_k, int batch, long long total_q, int Hq, int Hkv, int d, int k,
                               float scale, void* O, float* lse, cudaStream_t stream, const uint8_t* skip_rows);

// Sparse attention of the selected sets with adjacent-query reuse: the union plan per 16-row
// block, the two masked tensor-core passes in their union form over the blocks whose union
// has at most max_chunks x 128 positions, and the gather kernel for the other rows.  Same O
// and lse as the gather kernel (within the same rounding bound).
int sa_block_reuse_launch(const void* Q, const void* K, const void* V, const int* indices, const int* cu_q,
                          const int* cu_k, int batch, long long total_q, long long total_k, int Hq, int Hkv, int k,
                          int max_seqlen_k, int max_chunks, float scale, void* O, float* lse, void* ws,
                          int* ucount_out, cudaStream_t s) {
  using C = dsa::SAFwdTcCfg;
  const SAUnionWs W = sa_union_layout(ws, total_q, Hq, batch, max_seqlen_k, max_chunks);
  const int words = (max_seqlen_k + 31) / 32;
  const int plan_smem = (2 * words + W.ucap / 128 * 64) * 4;
  if (const int st = sa_fwd_tc_setup(); st != DSA_OK) return st;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sa_union_plan_kernel,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  if (total_q <= 0) return DSA_OK;
  if (plan_smem > 200 * 1024) return DSA_ERR_UNSUPPORTED;
  int* ucount = ucount_out ? ucount_out : W.ucount;
  dsa::SAUnionPlanParams pp;
  pp.indices = indices;
  pp.k = k;
  pp.cu_q = cu_q;
  pp.cu_k = cu_k;
  pp.batch = batch;
  pp.ucap = W.ucap;
  pp.ukeys = W.ukeys;
  pp.ucount = ucount;
  pp.umask = W.umask;
  pp.blk_use = W.blk_use;
  pp.row_tc = W.row_tc;
  pp.blk_list = W.blk_list;
  pp.n_used = W.n_used;
  pp.max_union_frac = kUnionMaxFrac;
  const long long n_blocks = (total_q + 15) / 16 + batch;
  // blocks past the last sequence's end keep these zero: no union-form item, no count
  if (const cudaError_t e_ = cudaMemsetAsync(W.blk_use, 0, (size_t)n_blocks, s); e_ != cudaSuccess) return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemsetAsync(ucount, 0, (size_t)n_blocks * 4, s); e_ != cudaSuccess)
    return cuda_fail(e_);
  if (const cudaError_t e_ = cudaMemsetAsync(W.n_used, 0, 4, s); e_ != cudaSuccess) return cuda_fail(e_);
  dsa::sa_union_plan_kernel<<<(unsigned)n_blocks, dsa::SA_PLAN_T, plan_smem, s>>>(pp, words);
  if (const int st = last_launch_status(); st != DSA_OK) return st;
  KlUnion un{W.ukeys, ucount, W.umask, W.blk_use, W.ucap, W.blk_list, W.n_used};
  const float scale_log2 = scale * 1.4426950408889634f;
  int st = kl_lse_tc_launch(Q, K, cu_q, cu_k, batch, total_q, total_k, Hq, Hkv, 0, scale_log2, lse, s, nullptr,
                            0.69314718055994531f, W.mx, &un);
  if (st != DSA_OK) return st;
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)total_q};
    const uint64_t strides[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 8, 16};
    if (const int e = make_tmap_bf16_3d(&tq, Q, dims, strides, box); e != DSA_OK) return e;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)std::max<long long>(total_k, 1)};
    const uint64_t strides[2] = {256, (uint64_t)Hkv * 256};
    const uint32_t box[3] = {64, 1, 128};
    if (const int e = make_tmap_bf16_3d(&tk, K, dims, strides, box); e != DSA_OK) return e;
    if (const int e = make_tmap_bf16_3d(&tv, V, dims, strides, box); e != DSA_OK) return e;
  }
  dsa::SAFwdTcParams p{};
  p.items.cu_q = cu_q;
  p.items.cu_k = cu_k;
  p.items.batch = batch;
  p.items.Hq = Hq;
  p.items.Hkv = Hkv;
  p.items.scale_log2 = scale_log2;
  p.items.lse_out = lse;
  p.items.out_scale = 1.f;
  p.items.n_blocks = n_blocks;
  p.items.n_items = n_blocks * Hkv;
  p.items.mask = nullptr;
  p.items.total_q = total_q;
  p.items.max_out = nullptr;
  p.items.ukeys = W.ukeys;
  p.items.ucount = ucount;
  p.items.umask = W.umask;
  p.items.blk_use = W.blk_use;
  p.items.ucap = W.ucap;
  p.items.blk_list = W.blk_list;
  p.items.n_used = W.n_used;
  p.items.K = static_cast<const uint16_t*>(K);
  p.K = static_cast<const uint16_t*>(K);
  p.V = static_cast<const uint16_t*>(V);
  p.lse = lse;
  p.mx = W.mx;
  p.O = static_cast<uint16_t*>(O);
  const long long grid = std::min<long long>(p.items.n_items, (long long)sm_count());
  dsa::sa_fwd_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, tv, p);
  if (last_launch_status() != DSA_OK) return DSA_ERR_CUDA;
  // the rows of the other blocks on the gather kernel
  return sparse_attn_prefill_launch(Q, K, V, indices, cu_q, cu_k, batch, total_q, Hq, Hkv, 128, k, scale, O, lse, s,
                                    W.row_tc);
}

}  // namespace dsa_host
