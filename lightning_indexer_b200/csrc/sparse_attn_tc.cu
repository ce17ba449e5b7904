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
// (bf16 in [0, 1], the largest exactly 1; written to shared memory in the 128-byte swizzled
// K-major layout), accumulates O += P . V_tile in TMEM with V read MN-major, and divides by
// the row sum 2^(lse - m) in fp32 at the end.  Knowing m first removes the running rescale
// of O.  Warps: 0 TMA, 1 MMA issuer and TMEM owner, 2-9 epilogue (two per TMEM lane
// quarter, one per 64-key half of each tile).
#include <algorithm>

#include "common.cuh"

namespace dsa {

struct SAFwdTcParams {
  KlLseParams items;      // work items (shared with the LSE pass)
  const uint32_t* mask;   // selection words, layout of KlLseParams::mask
  long long total_q;
  const float* lse;       // [T, Hq] natural log (first pass)
  const float* mx;        // [T, Hq] row maxima of the scaled logits, base 2 (first pass)
  uint16_t* O;            // [T, Hq, 128] bf16
};

struct SAFwdTcCfg {
  static constexpr int TILE_BYTES = 128 * 128 * 2;
  static constexpr int PANEL_BYTES = 128 * 128;
  // K tiles are free after their S MMA, V tiles only after P.V: separate rings, the K ring
  // one deeper so the next tiles' keys load while the epilogue works
  static constexpr int K_STAGES = 3, V_STAGES = 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + TILE_BYTES;
  static constexpr int OFF_V = OFF_K + K_STAGES * TILE_BYTES;
  static constexpr int OFF_P = OFF_V + V_STAGES * TILE_BYTES;
  static constexpr int OFF_BAR = OFF_P + TILE_BYTES;
  // q_full, q_empty, k_full[K], k_empty[K], v_full[V], v_empty[V], s_full[2], s_empty[2],
  // p_full, p_empty, o_full, o_empty, done
  static constexpr int NUM_BARS = 2 + 2 * K_STAGES + 2 * V_STAGES + 4 + 2 + 2 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
  static constexpr int EPI_WARPS = 8;
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int TMEM_COLS = 512;  // S [0,128) [128,256), O [256,384)
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
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < C::V_STAGES; ++i) {
      mbar_init(&v_full[i], 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      long long m = 0, n = 0;    // items with key tiles, key tiles
      long long nk = 0, nv = 0;  // K and V tile copies issued (they differ after an abort)
      bool ok = true;
      for (long long item = blockIdx.x; item < ip.n_items && ok; item += gridDim.x) {
        KlLseItem it;
        if (!kl_lse_item(item, ip, it) || it.ntiles == 0) continue;
        if (!(ok = mbar_wait(q_empty, (uint32_t)(m & 1) ^ 1u, abort_flag, 120))) break;
        mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(smem + C::OFF_Q + pn * C::PANEL_BYTES, &tmap_q, q_full, pn * 64, it.g * G, (int)it.t0);
        ++m;
        for (int j = 0; j < it.ntiles; ++j, ++n) {
          const int ks = (int)(n % C::K_STAGES), vs = (int)(n % C::V_STAGES);
          if (!(ok = mbar_wait(&k_empty[ks], (uint32_t)((n / C::K_STAGES) & 1) ^ 1u, abort_flag, 121))) break;
          mbar_arrive_expect_tx(&k_full[ks], C::TILE_BYTES);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(smem + C::OFF_K + ks * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmap_k, &k_full[ks], pn * 64,
                        it.g, it.kbase + j * 128);
          ++nk;
          if (!(ok = mbar_wait(&v_empty[vs], (uint32_t)((n / C::V_STAGES) & 1) ^ 1u, abort_flag, 130))) break;
          mbar_arrive_expect_tx(&v_full[vs], C::TILE_BYTES);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(smem + C::OFF_V + vs * C::TILE_BYTES + pn * C::PANEL_BYTES, &tmap_v, &v_full[vs], pn * 64,
                        it.g, it.kbase + j * 128);
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
      const uint32_t p_base = smem_u32(smem + C::OFF_P);
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
      for (long long item = blockIdx.x; item < ip.n_items && ok; item += gridDim.x) {
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
          for (int kk = 0; kk < 8; ++kk)  // K = 128 keys, 16 per step
            umma_bf16(tmem_base + 256,
                      smem_desc_kmajor(p_base + (kk / 4) * C::PANEL_BYTES + (kk % 4) * 32, 128),
                      smem_desc_mn_sw128(v_base + kk * 16 * 128, C::PANEL_BYTES), C::IDESC_O, (j | kk) != 0);
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
    // ------------------------------------------------------------ epilogue (8 warps)
    const int quarter = warp % 4;
    const int half = (warp - 2) / 4;    // keys 64 half .. 64 half + 63 of each tile; O dims likewise
    const int r = quarter * 32 + lane;  // (token, head) of this lane: token r / 8, head r % 8
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const uint32_t p_row = smem_u32(smem + C::OFF_P) + half * C::PANEL_BYTES + r * 128;
    long long m = 0, n = 0;
    bool ok = true;
    for (long long item = blockIdx.x; item < ip.n_items && ok; item += gridDim.x) {
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
      const uint32_t* mrow = p.mask + (it.t0 + (valid ? u : 0)) * 4 + 2 * half;
      for (int j = 0; j < it.ntiles; ++j, ++n) {
        const int sb = (int)(n & 1);
        uint32_t w0 = 0u, w1 = 0u;
        if (valid) {
          w0 = mrow[(long long)j * p.total_q * 4];
          w1 = mrow[(long long)j * p.total_q * 4 + 1];
        }
        if (!(ok = mbar_wait(&s_full[sb], (uint32_t)((n >> 1) & 1), abort_flag, 127))) break;
        tc_fence_after();
        float x[64];
        tmem_ld_x32_sync(tmem_base + lane_off + sb * 128 + half * 64, x);
        tmem_ld_x32_sync(tmem_base + lane_off + sb * 128 + half * 64 + 32, x + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
        uint32_t pk[32];
#pragma unroll
        for (int c = 0; c < 64; c += 2) {
          const uint32_t w = c < 32 ? w0 : w1;
          const float p0 = ((w >> (c & 31)) & 1u) ? ex2_ftz(fmaf(x[c], ip.scale_log2, nl)) : 0.f;
          const float p1 = ((w >> ((c + 1) & 31)) & 1u) ? ex2_ftz(fmaf(x[c + 1], ip.scale_log2, nl)) : 0.f;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[c / 2] = *reinterpret_cast<uint32_t*>(&b2);
        }
        if (!(ok = mbar_wait(p_empty, (uint32_t)(n & 1) ^ 1u, abort_flag, 128))) break;
#pragma unroll
        for (int q = 0; q < 8; ++q)  // 16-byte chunk q of this row's panel: keys 8q .. 8q+7
          asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(p_row + ((q ^ (r & 7)) * 16)),
                       "r"(pk[4 * q]), "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                       : "memory");
        fence_proxy_async_shared();  // the tensor core reads P through the async proxy
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(o_full, (uint32_t)(m & 1), abort_flag, 129))) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 64; c += 32) {
        float v[32];
        tmem_ld_x32_sync(tmem_base + lane_off + 256 + half * 64 + c, v);
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
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

namespace dsa_host {

int kl_lse_tc_launch(const void* Q, const void* K, const int* cu_q, const int* cu_k, int batch, long long T,
                     long long Tk, int Hq, int Hkv, int max_seqlen_q, float scale_log2, float* lse_out,
                     cudaStream_t s, const uint32_t* mask, float out_scale, float* max_out);

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
  static DeviceFlag attr_done;
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(dsa::sa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    C::SMEM_BYTES);
        e_ != cudaSuccess)
      return cuda_fail(e_);
    attr_done = true;
  }
  if (total_q <= 0) return DSA_OK;
  uint32_t* mask = static_cast<uint32_t*>(mask_ws);
  float* mx = reinterpret_cast<float*>(static_cast<uint8_t*>(mask_ws) + sa_fwd_tc_mask_only(total_q, max_seqlen_k));
  int st = sa_bwd_mask_build(indices, cu_q, cu_k, batch, total_q, k, max_seqlen_k, mask, s);
  if (st != DSA_OK) return st;
  const float scale_log2 = scale * 1.4426950408889634f;
  st = kl_lse_tc_launch(Q, K, cu_q, cu_k, batch, total_q, total_k, Hq, Hkv, 0, scale_log2, lse, s, mask,
                        0.69314718055994531f, mx);
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
  dsa::SAFwdTcParams p;
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
  p.mask = mask;
  p.total_q = total_q;
  p.lse = lse;
  p.mx = mx;
  p.O = static_cast<uint16_t*>(O);
  const long long grid = std::min<long long>(p.items.n_items, (long long)sm_count());
  dsa::sa_fwd_tc_kernel<<<(unsigned)grid, C::THREADS, C::SMEM_BYTES, s>>>(tq, tk, tv, p);
  return last_launch_status();
}

}  // namespace dsa_host
