// Dense attention of the KL target on tcgen05 tensor cores (sm_100a): the LSE pass and the
// target / KL / gradient pass.
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: the dense warm-up
// trains the indexer against the full attention distribution; its target needs, for every
// query row t and head h, the log-sum-exp of the dense causal logits
//   lse[t,h] = log sum_{s visible to t} exp(scale * Q[t,h] . K[s, h / (Hq/Hkv)]),
// kept in base 2 (lse / ln 2) for the exp2-based passes that read it.
//
// One work item is (16 query rows of one sequence, one KV head g): the A operand is the
// 16 rows x 8 query heads of group g (M = 128, read by a 3-D TMA box straight from
// Q [T, Hq, d]), the B operand a tile of 128 keys of K [Tk, Hkv, d] (3-D box, head g),
// K = d = 128.  Each TMEM lane is one (row, head), so the online log-sum-exp over the keys
// is thread-local in the epilogue.  Persistent CTAs, warp-specialised: warp 0 TMA, warp 1
// MMA issuer and TMEM owner, warps 2-9 epilogue (two per TMEM lane quarter, one per
// 64-key half of each tile; their two running (max, sum) pairs merge at the item's end);
// two accumulator buffers, six key stages.
//
// Union form (adjacent-query reuse, report summary section 8): a block visits, instead of
// its causal key tiles, chunks of 128 positions of the sorted union of its rows' selected
// sets; two gather warps copy those K rows into the swizzled tile with 16-byte cp.async
// (each warp instruction reads two whole 256-byte rows), and the per-(row, union slot)
// selection bits mask S.
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct KlLseParams {
  const int* cu_q;
  const int* cu_k;
  int batch;
  int Hq, Hkv;
  float scale_log2;
  float* lse_out;  // [T, Hq]: base-2 log times out_scale
  float out_scale;     // 1 (base 2) or ln 2 (natural log)
  long long n_blocks;  // 16-row blocks over all sequences
  long long n_items;   // n_blocks * Hkv
  // optional selection: only keys whose bit is set count (bit s % 32 of word
  // ((s / 128) * T + t) * 4 + (s % 128) / 32); blocks with no visible key are kept then,
  // so that their rows get -inf
  const uint32_t* mask;
  long long total_q;
  float* max_out;  // optional [T, Hq]: the row maxima of the scaled logits in base 2
  // optional union form: only blocks with blk_use[blk] != 0 are items (blk: the block's
  // number in ascending order over the sequences); block blk visits ceil(ucount[blk] / 128)
  // chunks of the positions ukeys[blk * ucap ..] (sequence-local, ascending, padded with
  // position 0 to a whole chunk), with selection words
  // umask[((blk * (ucap / 128) + chunk) * 16 + row) * 4 + slot / 32] (bit slot % 32) in
  // place of `mask`; the key tensor map then addresses K as rows (s * Hkv + g) of d values
  const int* ukeys = nullptr;
  const int* ucount = nullptr;
  const uint32_t* umask = nullptr;
  const uint8_t* blk_use = nullptr;
  int ucap = 0;
  const uint16_t* K = nullptr;  // union form: K [Tk, Hkv, 128] bf16, read by the gather warps
  // union form: the union-form blocks (item i is block blk_list[i / Hkv], head i % Hkv) and
  // their number, so that the passes visit no other block
  const int* blk_list = nullptr;
  const int* n_used = nullptr;
};

struct KlLseItem {
  long long t0;
  int ntok, i0, Lq, Lk, kbase, g, ntiles;
  long long blk;
};

// item -> (block, head); blocks are numbered from the last (usually the longest rows)
// The number of items of a launch: every (block, KV head), or the union form's listed ones.
__device__ __forceinline__ long long kl_item_count(const KlLseParams& p) {
  return p.blk_list ? (long long)__ldg(p.n_used) * p.Hkv : p.n_items;
}

__device__ __forceinline__ bool kl_lse_item(long long item, const KlLseParams& p, KlLseItem& it) {
  it.g = (int)(item % p.Hkv);
  long long r = p.blk_list ? __ldg(p.blk_list + item / p.Hkv) : p.n_blocks - 1 - item / p.Hkv;
  it.blk = r;
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
      if (p.ukeys) {
        if (!p.blk_use[it.blk]) return false;
        it.ntiles = (__ldg(p.ucount + it.blk) + 127) / 128;
        return true;
      }
      return it.ntiles > 0 || p.mask != nullptr;
    }
    r -= nb;
  }
  return false;
}

// Union form: the 128 rows (positions chunk_keys[0..127], sequence-local; head g of a
// [Tk, Hkv, 128] bf16 tensor) of one union chunk copied into a K-major tile with the
// 128-byte swizzle (two 64-column panels of 128-byte rows, 16-byte chunk c of row r at
// ((c ^ (r % 8)) * 16)), the layout a tiled TMA load gives.  Called by `nw` gather warps
// (wg = 0 .. nw-1).  Eight lanes per row: each warp instruction moves the 128-byte halves of
// four rows (whole lines, as coalesced as two full rows per instruction), and a row's
// position and address are worked out once for both halves.  Every lane then arrives on
// `bar` when its copies have landed (nw * 32 arrivals).
__device__ __forceinline__ void union_copy_tile(uint8_t* dst, int panel_bytes, const uint16_t* src,
                                                const int* chunk_keys, int kbase, int Hkv, int g, int nw, int wg,
                                                int lane, uint64_t* bar) {
  const int sub = lane >> 3, c = lane & 7;
  const uint32_t dbase = smem_u32(dst);
  const uint16_t* base = src + (long long)g * 128 + c * 8;
  const long long stride = (long long)Hkv * 128;
#pragma unroll 2
  for (int q = wg; q < 32; q += nw) {
    const int r = 4 * q + sub;
    const int s = __ldg(chunk_keys + r);  // eight lanes read each position (one L1 line per chunk)
    const uint16_t* row = base + (long long)(kbase + s) * stride;
    const uint32_t d0 = dbase + r * 128 + ((c ^ (r & 7)) * 16);
    cp_async_16(d0, row, true);                     // columns 8c .. 8c + 7 (panel 0)
    cp_async_16(d0 + panel_bytes, row + 64, true);  // columns 64 + 8c .. (panel 1)
  }
  cp_async_mbar_arrive(bar);
}

// One row's two selection words (a 64-key half) per tile, loaded two tiles ahead of their use:
// their global-memory latency would otherwise stall the epilogue at every tile.  Without a
// row (no selection, or a row past the block's tokens) every word is `fill`.
struct MaskWords {
  const uint32_t* row;
  long long stride;
  int n;
  uint32_t fill;
  uint2 a, b;  // the words of tiles j and j + 1
  __device__ __forceinline__ MaskWords(const uint32_t* r, long long s, int ntiles, uint32_t f)
      : row(r), stride(s), n(ntiles), fill(f) {
    a = load(0);
    b = load(1);
  }
  __device__ __forceinline__ uint2 load(int j) const {
    return (row && j < n) ? make_uint2(row[(long long)j * stride], row[(long long)j * stride + 1]) : make_uint2(fill, fill);
  }
  // the words of tile j (called with j = 0, 1, 2, ... in order)
  __device__ __forceinline__ uint2 next(int j) {
    const uint2 w = a;
    a = b;
    b = load(j + 2);
    return w;
  }
};

// The selection words of row u of an item and the distance between its tiles' (or union
// chunks') words: the union form's per-block words, else the full layout of `mask`, else
// none.  Rows past the block's tokens read row 0's words (they are masked anyway).
__device__ __forceinline__ const uint32_t* kl_mask_row(const KlLseParams& p, const KlLseItem& it, int u,
                                                       long long& stride) {
  if (p.ukeys) {
    stride = 64;
    return p.umask + (it.blk * (p.ucap / 128) * 16 + u) * 4;
  }
  stride = p.total_q * 4;
  return p.mask ? p.mask + (it.t0 + u) * 4 : nullptr;
}

struct KlLseCfg {
  static constexpr int TILE_BYTES = 128 * 128 * 2;
  static constexpr int PANEL_BYTES = 128 * 128;
  static constexpr int B_STAGES = 6;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + TILE_BYTES;
  static constexpr int OFF_BAR = OFF_B + B_STAGES * TILE_BYTES;
  // a_full, a_empty, b_full[S], b_empty[S], acc_full[2], acc_empty[2], done, ml_full, ml_empty
  static constexpr int NUM_BARS = 2 + 2 * B_STAGES + 4 + 1 + 2;
  static constexpr int OFF_ML = OFF_BAR + NUM_BARS * 8;  // 128 (max, sum) pairs of the second half
  static constexpr int OFF_MISC = OFF_ML + 128 * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  // Warps: 0 TMA, 1 MMA and TMEM, 2-3 gather (warpgroup 0); 4-11 epilogue (warpgroups 1-2);
  // 12-15 gather (warpgroup 3).  The six gather warps copy the union form's key chunks with
  // cp.async and idle otherwise.  Registers after the reallocation: 80 for warpgroup 0, 152
  // for the epilogue, 64 for warpgroup 3 (128 x (80 + 64) + 256 x 152 = 57344 of the 65536
  // that 512 threads at 128 registers hold).
  static constexpr int EPI_WARPS = 8;
  static constexpr int GATHER_WARPS = 6;
  static constexpr int THREADS = 512;
  static constexpr int REG_WG0 = 80, REG_EPI = 152, REG_WG3 = 64;
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
  uint64_t* ml_full = acc_full + 5;
  uint64_t* ml_empty = acc_full + 6;
  float2* sML = reinterpret_cast<float2*>(smem + C::OFF_ML);
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int i = 0; i < C::B_STAGES; ++i) {
      // a key tile lands by TMA (one arrival with its bytes), or in the union form by the
      // gather warps' cp.async (one arrival per gather thread)
      mbar_init(&b_full[i], p.ukeys ? C::GATHER_WARPS * 32 : 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    mbar_init(ml_full, C::EPI_WARPS / 2);
    mbar_init(ml_empty, C::EPI_WARPS / 2);
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
  const long long n_items = kl_item_count(p);

  // ------------------------------------------------------------ gather warps (union form),
  // in warpgroups 0 and 3: warps 2-3 and 12-15
  auto gather_role = [&]() {
    if (p.ukeys) {
      const int wg = warp < 4 ? warp - 2 : warp - 10;
      long long n = 0;
      bool ok = true;
      for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        KlLseItem it;
        if (!kl_lse_item(item, p, it)) continue;
        const int* keys = p.ukeys + it.blk * p.ucap;
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int st = (int)(n % C::B_STAGES);
          if (lane == 0) ok = mbar_wait(&b_empty[st], (uint32_t)((n / C::B_STAGES) & 1) ^ 1u, abort_flag, 68);
          if (!(ok = __shfl_sync(0xffffffffu, ok, 0))) break;
          union_copy_tile(sB + st * C::TILE_BYTES, C::PANEL_BYTES, p.K, keys + j * 128, it.kbase, p.Hkv, it.g,
                          C::GATHER_WARPS, wg, lane, &b_full[st]);
        }
      }
      cp_async_wait<0>();  // nothing of this thread's in flight when the CTA leaves
    }
  };
  if (warp < 4) {
    setmaxnreg_dec<C::REG_WG0>();
    if (warp == 0) {
      // ------------------------------------------------------------ TMA producer (the query
      // block of each item; the key tiles too, except in the union form)
      if (lane == 0) {
        long long m = 0, n = 0;  // items, key tiles
        bool ok = true;
        for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
          KlLseItem it;
          if (!kl_lse_item(item, p, it)) continue;
          if (!(ok = mbar_wait(a_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 60))) break;
          mbar_arrive_expect_tx(a_full, C::TILE_BYTES);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(sA + pn * C::PANEL_BYTES, &tmap_q, a_full, pn * 64, it.g * G, (int)it.t0);
          ++m;
          if (p.ukeys) continue;  // the gather warps copy the union chunks
          for (int j = 0; j < it.ntiles; ++j) {
            const int st = (int)(n % C::B_STAGES);
            if (!(ok = mbar_wait(&b_empty[st], (uint32_t)((n / C::B_STAGES) & 1) ^ 1u, abort_flag, 61))) break;
            mbar_arrive_expect_tx(&b_full[st], C::TILE_BYTES);
            for (int pn = 0; pn < 2; ++pn)
              tma_load_3d(sB + st * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmap_k, &b_full[st], pn * 64, it.g,
                          it.kbase + j * 128);
            ++n;
          }
        }
        if (!ok) {
          // let the copies issued so far land before the CTA exits (bounded)
          uint64_t t0 = globaltimer_ns();
          for (long long q = max(0LL, n - C::B_STAGES); q < n; ++q)
            while (!mbar_try_wait(smem_u32(&b_full[q % C::B_STAGES]), (uint32_t)((q / C::B_STAGES) & 1)) &&
                   globaltimer_ns() - t0 < 100000000ull) {
            }
          t0 = globaltimer_ns();
          if (m > 0)
            while (!mbar_try_wait(smem_u32(a_full), (uint32_t)((m - 1) & 1)) && globaltimer_ns() - t0 < 100000000ull) {
            }
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        long long m = 0, n = 0;
        bool ok = true;
        const uint32_t a_base = smem_u32(sA);
        for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
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
      gather_role();
    }
  } else if (warp < 4 + C::EPI_WARPS) {
    setmaxnreg_inc<C::REG_EPI>();
    // ------------------------------------------------------------ epilogue (8 warps)
    const int lane_grp = warp % 4;
    const int half = (warp - 4) / 4;     // keys 64 half .. 64 half + 63 of each tile
    const int r = lane_grp * 32 + lane;  // (row, head) of this thread: row r / 8, head r % 8
    const uint32_t lane_off = (uint32_t)(lane_grp * 32) << 16;
    long long n = 0, m = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      KlLseItem it;
      if (!kl_lse_item(item, p, it)) continue;
      const int u = r / 8;
      const bool valid = u < it.ntok;
      // (union chunks hold only positions that the rows selecting them can see)
      const int vis = valid ? (p.ukeys ? INT_MAX : causal_vis(it.i0 + u, it.Lq, it.Lk)) : 0;
      // running max of the raw logits and sum of 2^(scale (x - max)) (scale > 0)
      float mx = -INFINITY, l = 0.f;
      long long mstride;
      const uint32_t* mrow = kl_mask_row(p, it, valid ? u : 0, mstride);
      if (mrow) mrow += 2 * half;
      // selection words of this row for the half's 64 keys (all set without a selection)
      MaskWords mw(mrow, mstride, it.ntiles, 0xffffffffu);
      for (int j = 0; j < it.ntiles; ++j, ++n) {
        const int tile = j;
        const int ab = (int)(n & 1);
        const uint2 wj = mw.next(j);
        const uint32_t w0 = wj.x, w1 = wj.y;
        if (!(ok = mbar_wait(&acc_full[ab], (uint32_t)((n >> 1) & 1), abort_flag, 65))) break;
        tc_fence_after();
        float v[64];
        tmem_ld_x32_sync(tmem_base + lane_off + ab * 128 + half * 64, v);
        tmem_ld_x32_sync(tmem_base + lane_off + ab * 128 + half * 64 + 32, v + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        const int nvis = vis == INT_MAX ? 64 : vis - (tile * 128 + half * 64);  // keys of this half the row sees
        if (nvis < 64) {
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (q >= nvis) v[q] = -INFINITY;
        }
        if ((w0 & w1) != 0xffffffffu) {
#pragma unroll
          for (int q = 0; q < 64; ++q)
            if (!(((q < 32 ? w0 : w1) >> (q & 31)) & 1u)) v[q] = -INFINITY;
        }
        float cm = v[0];
#pragma unroll
        for (int q = 1; q < 64; ++q) cm = fmaxf(cm, v[q]);
        if (cm > mx) {
          l *= ex2_ftz((mx - cm) * p.scale_log2);  // mx = -inf: l is 0
          mx = cm;
        }
        if (mx > -INFINITY) {
          const float nb = -mx * p.scale_log2;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int q = 0; q < 64; q += 4) {
            a0 += ex2_ftz(fmaf(v[q], p.scale_log2, nb));
            a1 += ex2_ftz(fmaf(v[q + 1], p.scale_log2, nb));
            a2 += ex2_ftz(fmaf(v[q + 2], p.scale_log2, nb));
            a3 += ex2_ftz(fmaf(v[q + 3], p.scale_log2, nb));
          }
          l += (a0 + a1) + (a2 + a3);
        }
      }
      if (!ok) break;
      // merge the two halves: (mx, l) of keys 64..127 of each tile into those of 0..63
      if (half == 1) {
        if (!(ok = mbar_wait(ml_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 66))) break;
        sML[r] = make_float2(mx, l);
        __syncwarp();
        if (lane == 0) mbar_arrive(ml_full);
      } else {
        if (!(ok = mbar_wait(ml_full, (uint32_t)(m & 1), abort_flag, 67))) break;
        const float2 o = sML[r];
        __syncwarp();
        if (lane == 0) mbar_arrive(ml_empty);
        const float M = fmaxf(mx, o.x);
        float L = 0.f;
        if (M > -INFINITY) L = l * ex2_ftz((mx - M) * p.scale_log2) + o.y * ex2_ftz((o.x - M) * p.scale_log2);
        if (valid) {
          const long long o = (it.t0 + u) * p.Hq + it.g * G + (r % 8);
          p.lse_out[o] = L > 0.f ? (M * p.scale_log2 + log2f(L)) * p.out_scale : -INFINITY;
          if (p.max_out) p.max_out[o] = L > 0.f ? M * p.scale_log2 : -INFINITY;
        }
      }
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


// ---------------------------------------------------------------------------- target
// Dense target p, the row's KL term and g = dloss/dI for the rows [row_begin, row_end) of
// one score chunk (same source and definitions as the LSE above):
//   p[t,s]  = (1/Hq) sum_h exp(scale Q[t,h].K[s,g(h)] - lse[t,h])
//   kl[t]   = sum_{s visible} p (log p - log q),  log q = I[t,s] - lseI[t]
//   I[t,s] <- (q - p) / T   (in place)
// A work item is 8 query rows of one sequence.  Orientation is key-stationary per tile:
// the A operand is 128 keys of one KV head (M = 128), the B operand the 8 rows x 8 query
// heads of that KV head (N = 64, one 3-D TMA box of Q), so a TMEM lane is a key and the
// sum over heads stays inside a thread.  All Hkv (<= 4) heads of a key tile go to one
// 256-column TMEM buffer; two buffers alternate.  Sixteen epilogue warps: warp w reads lanes
// 32 (w % 4) .. (keys) for rows 2 ((w - 2) / 4) .. + 1.  Each (row, warp-quarter) keeps its
// own partial of kl[t], written once to kl_part[t][quarter] (a fixed-order sum follows).
struct KlTgtParams {
  const int* cu_q;
  const int* cu_k;
  int batch;
  int Hq, Hkv;
  float scale_log2;
  long long row_begin, row_end;
  const float* lse_att;  // [T, Hq] base-2 log
  const float* lseI;     // [row_end - row_begin]
  float* scores;         // [row_end - row_begin, ld]: I in, g out
  long long ld;
  float inv_T;
  float* kl_part;        // [T, 4]
  long long n_blocks;    // bound on the 8-row blocks of the chunk
  long long n_slots;     // n_blocks rounded up to whole rounds of gridDim.x
  // sparse-adaptation form: only the selected (t, s) pairs count (bit s & 31 of
  // mask[((s >> 7) * mask_rows + t) * 4 + ((s >> 5) & 3)]); the others get g = 0
  const uint32_t* mask = nullptr;
  long long mask_rows = 0;
};

struct KlTgtItem {
  long long t0;
  int ntok, i0, Lq, Lk, kbase, ntiles;
};

// Items in snake order over rounds of gridDim.x; within the order blocks run from the
// chunk's last one, so long rows come first.
__device__ __forceinline__ bool kl_tgt_item(long long item, const KlTgtParams& p, KlTgtItem& it) {
  RowBlock rb;
  if (!chunk_row_block<8>(snake_slot(item), p.cu_q, p.cu_k, p.batch, p.row_begin, p.row_end, p.n_blocks, rb))
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

struct KlTgtCfg {
  static constexpr int K_TILE_BYTES = 128 * 128 * 2;  // 128 keys x 128 dims
  static constexpr int K_PANEL_BYTES = 128 * 128;
  static constexpr int Q_GROUP_BYTES = 64 * 128 * 2;  // 8 rows x 8 heads x 128 dims
  static constexpr int Q_PANEL_BYTES = 64 * 128;
  static constexpr int MAX_HKV = 4;
  static constexpr int B_STAGES = 4;
  static constexpr int L_BYTES = 8 * 8 * MAX_HKV * 4;  // lse of 8 rows x Hq heads
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_B = OFF_Q + MAX_HKV * Q_GROUP_BYTES;
  static constexpr int OFF_L = OFF_B + B_STAGES * K_TILE_BYTES;
  static constexpr int OFF_BAR = OFF_L + 2 * L_BYTES;
  // q_full, q_empty, l_full[2], l_empty[2], b_full[S], b_empty[S], acc_full[2], acc_empty[2], done
  static constexpr int NUM_BARS = 2 + 4 + 2 * B_STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int EPI_WARPS = 16;
  static constexpr int ROWS_PER_WARP = 8 / (EPI_WARPS / 4);
  static_assert(ROWS_PER_WARP == 2, "one 16-column TMEM load per KV head and warp");
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int TMEM_COLS = 512;
  static constexpr int ACC_COLS = 256;
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, 64);
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

__global__ void __launch_bounds__(KlTgtCfg::THREADS, 1)
    kl_target_tc_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                        const KlTgtParams p) {
  using C = KlTgtCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sB = smem + C::OFF_B;
  float* sL = reinterpret_cast<float*>(smem + C::OFF_L);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* l_full = bars + 2;   // [2]
  uint64_t* l_empty = bars + 4;  // [2]
  uint64_t* b_full = bars + 6;   // [B_STAGES]
  uint64_t* b_empty = b_full + C::B_STAGES;
  uint64_t* acc_full = b_empty + C::B_STAGES;  // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2]
  uint64_t* mma_done = acc_full + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);
  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int Hkv = p.Hkv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&l_full[i], 1);
      mbar_init(&l_empty[i], C::EPI_WARPS);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_WARPS);
    }
    for (int i = 0; i < C::B_STAGES; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long m = 0, n = 0;  // items, (key tile, KV head) stages
      bool ok = true;
      for (long long item = blockIdx.x; item < p.n_slots && ok; item += gridDim.x) {
        KlTgtItem it;
        if (!kl_tgt_item(item, p, it)) continue;
        const int lb = (int)(m & 1);
        if (!(ok = mbar_wait(&l_empty[lb], (uint32_t)((m >> 1) & 1) ^ 1u, abort_flag, 70))) break;
        {
          const uint32_t lbytes = (uint32_t)(it.ntok * p.Hq * 4);
          mbar_arrive_expect_tx(&l_full[lb], lbytes);
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  smem_u32(sL + lb * (C::L_BYTES / 4))),
              "l"(p.lse_att + it.t0 * p.Hq), "r"(lbytes), "r"(smem_u32(&l_full[lb]))
              : "memory");
        }
        if (!(ok = mbar_wait(q_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 71))) break;
        mbar_arrive_expect_tx(q_full, Hkv * C::Q_GROUP_BYTES);
        for (int g = 0; g < Hkv; ++g)
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(sQ + g * C::Q_GROUP_BYTES + pn * C::Q_PANEL_BYTES, &tmap_q, q_full, pn * 64, g * 8,
                        (int)it.t0);
        ++m;
        for (int j = 0; j < it.ntiles && ok; ++j) {
          for (int g = 0; g < Hkv; ++g, ++n) {
            const int st = (int)(n % C::B_STAGES);
            if (!(ok = mbar_wait(&b_empty[st], (uint32_t)((n / C::B_STAGES) & 1) ^ 1u, abort_flag, 72))) break;
            mbar_arrive_expect_tx(&b_full[st], C::K_TILE_BYTES);
            for (int pn = 0; pn < 2; ++pn)
              tma_load_3d(sB + st * C::K_TILE_BYTES + pn * C::K_PANEL_BYTES, &tmap_k, &b_full[st], pn * 64, g,
                          it.kbase + j * 128);
          }
        }
      }
      if (!ok) {
        // let the copies this thread issued land before the CTA exits (bounded)
        const uint64_t t0 = globaltimer_ns();
        for (long long k = max(0LL, n - C::B_STAGES); k < n; ++k)
          while (!mbar_try_wait(smem_u32(&b_full[k % C::B_STAGES]), (uint32_t)((k / C::B_STAGES) & 1)) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        if (m > 0) {
          while (!mbar_try_wait(smem_u32(q_full), (uint32_t)((m - 1) & 1)) && globaltimer_ns() - t0 < 100000000ull) {
          }
          const long long k = m - 1;
          while (!mbar_try_wait(smem_u32(&l_full[k & 1]), (uint32_t)((k >> 1) & 1)) &&
                 globaltimer_ns() - t0 < 100000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      long long m = 0, n = 0, nt = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      for (long long item = blockIdx.x; item < p.n_slots && ok; item += gridDim.x) {
        KlTgtItem it;
        if (!kl_tgt_item(item, p, it)) continue;
        if (!(ok = mbar_wait(q_full, (uint32_t)(m & 1), abort_flag, 73))) break;
        tc_fence_after();
        for (int j = 0; j < it.ntiles && ok; ++j, ++nt) {
          const int ab = (int)(nt & 1);
          if (!(ok = mbar_wait(&acc_empty[ab], (uint32_t)((nt >> 1) & 1) ^ 1u, abort_flag, 74))) break;
          tc_fence_after();
          for (int g = 0; g < Hkv; ++g, ++n) {
            const int st = (int)(n % C::B_STAGES);
            if (!(ok = mbar_wait(&b_full[st], (uint32_t)((n / C::B_STAGES) & 1), abort_flag, 75))) break;
            tc_fence_after();
            const uint32_t k_base = smem_u32(sB + st * C::K_TILE_BYTES);
            const uint32_t d = tmem_base + ab * C::ACC_COLS + g * 64;
#pragma unroll
            for (int pn = 0; pn < 2; ++pn)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16(d, smem_desc_kmajor(k_base + pn * C::K_PANEL_BYTES + kk * 32, 128),
                          smem_desc_kmajor(q_base + g * C::Q_GROUP_BYTES + pn * C::Q_PANEL_BYTES + kk * 32, 128),
                          C::IDESC, (pn | kk) != 0);
            umma_commit(&b_empty[st]);
          }
          if (!ok) break;
          umma_commit(&acc_full[ab]);
        }
        if (!ok) break;
        umma_commit(q_empty);
        ++m;
      }
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (16 warps)
    constexpr int R = C::ROWS_PER_WARP;
    const int quarter = warp % 4;
    const int rgrp = (warp - 2) / 4;  // rows R rgrp .. R rgrp + R - 1
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float inv_Hq = 1.f / (float)p.Hq;
    long long m = 0, nt = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < p.n_slots && ok; item += gridDim.x) {
      KlTgtItem it;
      if (!kl_tgt_item(item, p, it)) continue;
      const int lb = (int)(m & 1);
      int vis[R];
      float lI[R], kl[R];
      float* Irow[R];
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        const int u = R * rgrp + rr;
        const bool valid = u < it.ntok;
        vis[rr] = valid ? causal_vis(it.i0 + u, it.Lq, it.Lk) : 0;
        const long long lr = it.t0 + (valid ? u : 0) - p.row_begin;
        lI[rr] = p.lseI[lr];
        Irow[rr] = p.scores + lr * p.ld;
        kl[rr] = 0.f;
      }
      if (!(ok = mbar_wait(&l_full[lb], (uint32_t)((m >> 1) & 1), abort_flag, 76))) break;
      const float* Lrow = sL + lb * (C::L_BYTES / 4) + R * rgrp * p.Hq;
      for (int j = 0; j < it.ntiles; ++j, ++nt) {
        const int ab = (int)(nt & 1);
        const int key = j * 128 + quarter * 32 + lane;
        float Iv[R];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) Iv[rr] = key < vis[rr] ? Irow[rr][key] : 0.f;
        if (!(ok = mbar_wait(&acc_full[ab], (uint32_t)((nt >> 1) & 1), abort_flag, 77))) break;
        tc_fence_after();
        float pr[R];
#pragma unroll
        for (int rr = 0; rr < R; ++rr) pr[rr] = 0.f;
        for (int g = 0; g < Hkv; ++g) {
          float v[8 * R];
          tmem_ld_x16_sync(tmem_base + lane_off + ab * C::ACC_COLS + g * 64 + rgrp * 8 * R, v);
#pragma unroll
          for (int rr = 0; rr < R; ++rr) {
            // 2^(scale log2(e) x - lse2) of the 8 heads of group g, summed
            const float4 La = *reinterpret_cast<const float4*>(Lrow + rr * p.Hq + g * 8);
            const float4 Lb = *reinterpret_cast<const float4*>(Lrow + rr * p.Hq + g * 8 + 4);
            const float* x = v + rr * 8;
            float a0 = ex2_ftz(fmaf(x[0], p.scale_log2, -La.x));
            float a1 = ex2_ftz(fmaf(x[1], p.scale_log2, -La.y));
            a0 += ex2_ftz(fmaf(x[2], p.scale_log2, -La.z));
            a1 += ex2_ftz(fmaf(x[3], p.scale_log2, -La.w));
            a0 += ex2_ftz(fmaf(x[4], p.scale_log2, -Lb.x));
            a1 += ex2_ftz(fmaf(x[5], p.scale_log2, -Lb.y));
            a0 += ex2_ftz(fmaf(x[6], p.scale_log2, -Lb.z));
            a1 += ex2_ftz(fmaf(x[7], p.scale_log2, -Lb.w));
            pr[rr] += a0 + a1;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
#pragma unroll
        for (int rr = 0; rr < R; ++rr) {
          if (key < vis[rr]) {
            bool sel = true;
            if (p.mask) {  // one word per (tile, row, lane quarter): the same for the whole warp
              const long long t = it.t0 + R * rgrp + rr;
              sel = (__ldg(p.mask + ((long long)j * p.mask_rows + t) * 4 + quarter) >> lane) & 1u;
            }
            if (sel) {
              const float pp = pr[rr] * inv_Hq;
              const float lq = Iv[rr] - lI[rr];  // log q
              if (pp > 0.f) kl[rr] += pp * (logf(pp) - lq);
              Irow[rr][key] = (expf(lq) - pp) * p.inv_T;
            } else {
              Irow[rr][key] = 0.f;
            }
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&l_empty[lb]);
      ++m;
#pragma unroll
      for (int rr = 0; rr < R; ++rr) {
        float s = kl[rr];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane == 0 && R * rgrp + rr < it.ntok) p.kl_part[(it.t0 + R * rgrp + rr) * 4 + quarter] = s;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// kl[t] = sum of its four key-quarter partials, in a fixed order
__global__ void kl_parts_sum_kernel(const float4* part, long long T, float* kl) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    const float4 v = part[t];
    kl[t] = ((v.x + v.y) + v.z) + v.w;
  }
}

}  // namespace dsa

namespace dsa_host {

// Dense LSE of every (row, head) for d = 128 and 8 query heads per KV head.
// lse_out = base-2 LSE times out_scale; with `mask`, over the selected keys only.
int kl_lse_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                     long long Tk, int Hq, int Hkv, int max_seqlen_q, float scale_log2, float* lse_out,
                     cudaStream_t s, const uint32_t* mask, float out_scale, float* max_out,
                     const KlUnion* un) {
  using C = dsa::KlLseCfg;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_lse_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    // the register reallocation must fit what a launch holds, or its increase would wait for
    // registers that never come
    cudaFuncAttributes fa;
    if (const cudaError_t e_ = cudaFuncGetAttributes(&fa, dsa::kl_lse_tc_kernel); e_ != cudaSuccess) return cuda_fail(e_);
    if ((long long)fa.numRegs * C::THREADS < 128LL * (C::REG_WG0 + C::REG_WG3) + 256LL * C::REG_EPI)
      return DSA_ERR_UNSUPPORTED;
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
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)std::max<long long>(Tk, 1)};
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
  p.out_scale = out_scale;
  p.mask = mask;
  p.total_q = T;
  p.max_out = max_out;
  if (un) {
    p.blk_list = un->blk_list;
    p.n_used = un->n_used;
    p.ukeys = un->ukeys;
    p.ucount = un->ucount;
    p.umask = un->umask;
    p.blk_use = un->blk_use;
    p.ucap = un->ucap;
    p.K = static_cast<const uint16_t*>(K);
  }
  // an upper bound on the 16-row blocks (each sequence rounds up once)
  p.n_blocks = (T + 15) / 16 + batch;
  p.n_items = p.n_blocks * Hkv;
  (void)max_seqlen_q;
  const long long grid = std::min<long long>(p.n_items, (long long)sm_count());
  if (grid <= 0) return DSA_OK;
  dsa::kl_lse_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, p);
  return last_launch_status();
}

// Dense target, kl partials and g for the chunk rows [r0, r1) (d = 128, Hq = 8 Hkv, Hkv <= 4).
int kl_target_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                        long long Tk, int Hq, int Hkv, long long r0, long long r1, float scale_log2,
                        const float* lse_att, const float* lseI, float* scores, long long ld, float inv_T,
                        float* kl_part, const uint32_t* mask, cudaStream_t s) {
  using C = dsa::KlTgtCfg;
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::kl_target_tc_kernel,
                                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  if (Hkv < 1 || Hkv > C::MAX_HKV || Hq != 8 * Hkv) return DSA_ERR_UNSUPPORTED;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[3] = {128, (uint64_t)Hq, (uint64_t)T};
    const uint64_t strides[2] = {256, (uint64_t)Hq * 256};
    const uint32_t box[3] = {64, 8, 8};
    if (const int st = make_tmap_bf16_3d(&tq, Q, dims, strides, box); st != DSA_OK) return st;
  }
  {
    const uint64_t dims[3] = {128, (uint64_t)Hkv, (uint64_t)Tk};
    const uint64_t strides[2] = {256, (uint64_t)Hkv * 256};
    const uint32_t box[3] = {64, 1, 128};
    if (const int st = make_tmap_bf16_3d(&tk, K, dims, strides, box); st != DSA_OK) return st;
  }
  dsa::KlTgtParams p;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.scale_log2 = scale_log2;
  p.row_begin = r0;
  p.row_end = r1;
  p.lse_att = lse_att;
  p.lseI = lseI;
  p.scores = scores;
  p.ld = ld;
  p.inv_T = inv_T;
  p.kl_part = kl_part;
  p.mask = mask;
  p.mask_rows = T;
  // an upper bound on the 8-row blocks (each sequence piece rounds up once)
  p.n_blocks = (r1 - r0 + 7) / 8 + batch;
  const long long grid = std::min<long long>(p.n_blocks, (long long)sm_count());
  if (grid <= 0) return DSA_OK;
  p.n_slots = (p.n_blocks + grid - 1) / grid * grid;
  dsa::kl_target_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, p);
  return last_launch_status();
}

int kl_parts_sum_launch(const float* kl_part, long long T, float* kl, cudaStream_t s) {
  if (T <= 0) return DSA_OK;
  dsa::kl_parts_sum_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(reinterpret_cast<const float4*>(kl_part), T,
                                                                       kl);
  return last_launch_status();
}

}  // namespace dsa_host
