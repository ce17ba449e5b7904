// Lightning-indexer scores on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// Same computation and epilogue as indexer.cu (Keye-VL-2.0 report summary,
// mqxn.cn/news/1966, section 1: MQA-shared lightning indexer), with the MMA spread over a
// pair of CTAs in a cluster of 2:
//   M = 256 keys per tile (128 from each CTA's shared memory),
//   N = NTOK tokens x H_I heads (each CTA holds the q_idx rows of half of the tokens),
//   D = 128 keys x N columns in each CTA's tensor memory.
// Per SM this halves the tensor core's B-operand reads from shared memory (each SM reads
// its 128 rows of A and N/2 rows of B per MMA instead of 128 + N), which is what the
// one-CTA kernel is bound by at N = 256.  The even CTA issues the MMAs; both CTAs load their
// own operand halves with TMA and run their own epilogue over their own 128 keys.
//   warp 0   TMA producer (both CTAs; completion counted on the even CTA's barriers)
//   warp 1   MMA issuer (even CTA only) + TMEM allocation (both, cta_group::2)
//   warps 2-3 idle (they complete warpgroup 0)
//   warps 4+ epilogue (both): tcgen05.ld -> fp32 ReLU/FMA over heads -> stores
// Warpgroup 0 gives registers up (setmaxnreg) to the epilogue warpgroups, whose per-thread
// state (head weights of two tokens, accumulators, candidate rings) needs more than an even
// split of the register file allows.
// Releases go back through multicast commits (stage free, accumulator full) to both CTAs
// and through remote arrivals (accumulator drained) to the even CTA.
//
// Three forms share the kernel (IndexerParams selects them):
//   - scores: every visible score is written to the fp32 score rows (dsa_index);
//   - sampled scores (key_stride S > 1): the keys are every S-th indexer key, so a row gets
//     about vis / S scores, from which the fused top-k takes a lower bound on the row's
//     k-th largest score;
//   - fused top-k (FUSED): no score is written; scores whose order key reaches the row's
//     bound are appended to the row's candidate list as (key, position).  Each epilogue
//     warp stages its candidates per token in a 64-entry shared-memory ring and moves 32
//     at a time to global memory behind one atomicAdd on the row's count; the add's result
//     is consumed only at the token's next key tile, so its round trip overlaps a tile of
//     work instead of stalling the warp.  The order of a row's list depends on timing; the
//     selection made from it does not.
#include "common.cuh"

namespace dsa {

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES, bool FUSED = false>
struct Indexer2Cfg {
  static constexpr int N = NTOK * H_I;  // MMA N over the pair
  static constexpr int NH = N / 2;      // q_idx rows held by each CTA
  static_assert(N % 32 == 0 && N >= 32 && N <= 256 && NTOK % 2 == 0, "pair UMMA N");
  static constexpr int PANEL = D_I >= 64 ? 64 : D_I;
  static constexpr int SWZ = PANEL * 2;
  static constexpr int NPANEL = D_I / PANEL;
  static constexpr int KSTEPS = PANEL / 16;
  static constexpr int A_BYTES = 128 * D_I * 2;
  static constexpr int B_BYTES = NH * D_I * 2;
  static constexpr int TMEM_COLS = (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr int EPI_THREADS = NUM_EPI_WARPS * 32;
  static constexpr int THREADS = 128 + EPI_THREADS;  // warpgroup 0 (roles), then the epilogue
  // registers per thread after the reallocation: warpgroup 0 / epilogue warpgroups.  With
  // 384 threads the launch holds 168 per thread (64512); 128 x 80 + 256 x 208 = 63488 fits,
  // and the 64-head epilogue then runs without spilling.
  static constexpr int REG_ROLE = 80;
  static constexpr int REG_EPI = 208;
  static_assert(NUM_EPI_WARPS % 4 == 0, "whole epilogue warpgroups");
  static constexpr int COL_PARTS = NUM_EPI_WARPS / 4;
  static constexpr int CPT = N / COL_PARTS;
  static_assert(CPT % H_I == 0 && H_I >= 32, "pair kernel epilogue: whole heads of whole tokens per thread");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + A_STAGES * A_BYTES;
  static constexpr int OFF_W = OFF_B + B_STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_W + 2 * N * 2;  // two bf16 weight buffers
  static constexpr int NUM_BARS = 2 * A_STAGES + 2 * B_STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  // fused form: a 64-entry (key, position) ring per epilogue warp and token it handles
  static constexpr int TPW = CPT / H_I;  // tokens per epilogue thread
  static constexpr int RING = 64;
  static constexpr int OFF_RING = OFF_MISC + 16;
  static constexpr int RING_BYTES = FUSED ? NUM_EPI_WARPS * TPW * RING * 8 : 0;
  static constexpr int SMEM_BYTES = OFF_RING + RING_BYTES + 1024;
  static constexpr uint32_t IDESC = idesc_bf16_f32(256, N);
  static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB per-block shared memory limit");
};

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES, bool FUSED>
__global__ void __launch_bounds__(Indexer2Cfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES, FUSED>::THREADS, 1)
    indexer2_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                    const IndexerParams p) {
  using C = Indexer2Cfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES, FUSED>;
  constexpr int TILE_KEYS = 256;
  // a repair pass with nothing to repair: both CTAs of every pair read the same flag and
  // leave before touching any barrier or tensor memory
  if (p.run_flag && *(volatile const int*)p.run_flag == 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;                                   // even CTA: both halves landed
  uint64_t* a_empty = bars + A_STAGES;                       // both CTAs: stage free
  uint64_t* b_full = bars + 2 * A_STAGES;                    // even CTA
  uint64_t* b_empty = bars + 2 * A_STAGES + B_STAGES;        // both CTAs
  uint64_t* acc_full = bars + 2 * A_STAGES + 2 * B_STAGES;   // both CTAs
  uint64_t* acc_empty = acc_full + 2;                        // even CTA: both epilogues drained
  uint64_t* mma_done = acc_full + 4;                         // even CTA
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();  // 0 = MMA-issuing CTA of the pair
  const long long pair = blockIdx.x / 2, npairs = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < A_STAGES; ++i) {
      mbar_init(&a_full[i], 1);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < B_STAGES; ++i) {
      mbar_init(&b_full[i], 1);
      mbar_init(&b_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 2 * NUM_EPI_WARPS);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc2(tmem_holder, C::TMEM_COLS);
    tmem_relinquish2();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmap_k);
    tma_prefetch_desc(&tmap_q);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised, TMEM of the pair allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp < 4) {
  setmaxnreg_dec<C::REG_ROLE>();  // the whole of warpgroup 0, before it splits into roles
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int as = 0, bs = 0;
      uint32_t aph = 0, bph = 0;
      bool ok = true;
      for (long long item = pair; item < p.n_items && ok; item += npairs) {
        Item it;
        if (!decode_item<NTOK, TILE_KEYS>(item, p, it)) continue;
        if (!(ok = mbar_wait(&b_empty[bs], bph ^ 1, abort_flag, 11))) break;
        if (rank == 0) mbar_arrive_expect_tx(&b_full[bs], 2 * C::B_BYTES);
        const uint32_t bfull = map_to_rank(&b_full[bs], 0);
        for (int pn = 0; pn < C::NPANEL; ++pn)
          tma_load_2d_pair(sB + bs * C::B_BYTES + pn * C::NH * C::SWZ, &tmap_q, bfull, pn * C::PANEL,
                           (int)((it.t0 + rank * (NTOK / 2)) * H_I));
        if (++bs == B_STAGES) { bs = 0; bph ^= 1; }
        for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
          if (!(ok = mbar_wait(&a_empty[as], aph ^ 1, abort_flag, 12))) break;
          if (rank == 0) mbar_arrive_expect_tx(&a_full[as], 2 * C::A_BYTES);
          const uint32_t afull = map_to_rank(&a_full[as], 0);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_2d_pair(sA + as * C::A_BYTES + pn * 128 * C::SWZ, &tmap_k, afull, pn * C::PANEL,
                             it.k0 + tile * TILE_KEYS + (int)rank * 128);
          if (++as == A_STAGES) { as = 0; aph ^= 1; }
        }
      }
      if (!ok && rank == 0) {
        for (int i = 0; i < A_STAGES; ++i) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(smem_u32(&a_full[i]), aph ^ (i >= as ? 1u : 0u)) &&
                 globaltimer_ns() - t0 < 200000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && rank == 0) {
      int as = 0, bs = 0, ab = 0;
      uint32_t aph = 0, bph = 0, abph = 0;
      bool ok = true;
      for (long long item = pair; item < p.n_items && ok; item += npairs) {
        Item it;
        if (!decode_item<NTOK, TILE_KEYS>(item, p, it)) continue;
        if (!(ok = mbar_wait(&b_full[bs], bph, abort_flag, 13))) break;
        const uint32_t b_base = smem_u32(sB + bs * C::B_BYTES);
        for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
          if (!(ok = mbar_wait(&acc_empty[ab], abph ^ 1, abort_flag, 14))) break;
          tc_fence_after();
          if (!(ok = mbar_wait(&a_full[as], aph, abort_flag, 15))) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + as * C::A_BYTES);
          const uint32_t d_tmem = tmem_base + ab * C::N;
#pragma unroll
          for (int pn = 0; pn < C::NPANEL; ++pn) {
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const uint64_t adesc = smem_desc_kmajor(a_base + pn * 128 * C::SWZ + kk * 32, C::SWZ);
              const uint64_t bdesc = smem_desc_kmajor(b_base + pn * C::NH * C::SWZ + kk * 32, C::SWZ);
              umma2_bf16(d_tmem, adesc, bdesc, C::IDESC, (pn | kk) != 0);
            }
          }
          umma2_commit_mc(&a_empty[as], 0x3);
          umma2_commit_mc(&acc_full[ab], 0x3);
          if (++as == A_STAGES) { as = 0; aph ^= 1; }
          if (++ab == 2) { ab = 0; abph ^= 1; }
        }
        if (!ok) break;
        umma2_commit_mc(&b_empty[bs], 0x3);
        if (++bs == B_STAGES) { bs = 0; bph ^= 1; }
      }
      umma2_commit_mc(mma_done, 0x1);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  }
  } else {
    setmaxnreg_inc<C::REG_EPI>();
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int ep = warp - 4;
    const int lane_grp = warp % 4;
    const int col_part = ep / 4;
    const int ep_tid = ep * 32 + lane;
    const int col0 = col_part * C::CPT;
    const uint32_t lane_off = (uint32_t)(lane_grp * 32) << 16;
    const uint32_t acc_empty0 = map_to_rank(&acc_empty[0], 0);
    const uint32_t acc_empty1 = map_to_rank(&acc_empty[1], 0);
    uint16_t* w_s = reinterpret_cast<uint16_t*>(sW);  // [2][N] bf16, the next item's prefetched
    // the head weights of an item (bf16, N values = N*2 bytes) go to w_s[buf] with 16-byte
    // asynchronous copies; rows past the block's valid tokens are copied too (never used)
    auto prefetch_w = [&](const Item& nx, int buf) {
      constexpr int CHUNKS = C::N * 2 / 16;
      if (ep_tid < CHUNKS) {
        const uint16_t* src = p.w + nx.t0 * H_I + ep_tid * 8;
        const bool valid = (nx.t0 * H_I + ep_tid * 8 + 8) <= p.w_elems;
        cp_async_16(smem_u32(w_s + buf * C::N + ep_tid * 8), valid ? src : p.w, valid);
      }
      cp_async_commit();
    };
    int ab = 0;
    uint32_t abph = 0;
    bool ok = true;
    int wbuf = 0;
    long long item = pair;
    Item it;
    bool have = false;
    for (; item < p.n_items; item += npairs)
      if ((have = decode_item<NTOK, TILE_KEYS>(item, p, it))) break;
    if (have) prefetch_w(it, 0);
    while (have && ok) {
      cp_async_wait<0>();
      named_bar_sync(1, C::EPI_THREADS);  // this item's weights landed; the other buffer is free
      // the next item this pair will see, and its weights in flight while this one runs
      Item nx;
      bool have_next = false;
      long long nitem = item + npairs;
      for (; nitem < p.n_items; nitem += npairs)
        if ((have_next = decode_item<NTOK, TILE_KEYS>(nitem, p, nx))) break;
      if (have_next) prefetch_w(nx, wbuf ^ 1);
      const int dvis = it.Lk - it.Lq + 1;
      // this thread's head weights for the whole item, two bf16 per register (a pair never
      // straddles two tokens: H_I is even); zero for rows past the block's tokens
      uint32_t wp[C::CPT / 2];
#pragma unroll
      for (int c = 0; c < C::CPT; c += 2) {
        const uint32_t pr = *reinterpret_cast<const uint32_t*>(w_s + wbuf * C::N + col0 + c);
        wp[c / 2] = (col0 + c) / H_I < it.ntok ? pr : 0u;
      }
      // visible keys (key-tensor-map rows) of this thread's tokens, 0 past the block's rows;
      // in the fused form also each token's bound and its ring state (warp-uniform)
      int vtok[C::TPW];
      // fused form, per token slot (warp-uniform): ring head, staged entries not yet
      // reserved, entries reserved by an atomicAdd whose result (pbase, lane 0) is consumed
      // only when the slot is next visited, so the add's round trip overlaps a key tile
      uint32_t thr_t[C::TPW], rhead[C::TPW], rcount[C::TPW], pend[C::TPW], pbase[C::TPW];
#pragma unroll
      for (int j = 0; j < C::TPW; ++j) {
        const int tok = col0 / H_I + j;
        vtok[j] = tok < it.ntok ? item_visible(p, it, min(max(it.i0 + tok + dvis, 0), it.Lk)) : 0;
        thr_t[j] = FUSED && tok < it.ntok ? __ldg(p.thr + (it.t0 + tok - p.row_begin) * p.state_ld) : 0xFFFFFFFFu;
        rhead[j] = 0;
        rcount[j] = 0;
        pend[j] = 0;
        pbase[j] = 0;
      }
      // reserves the oldest n (<= 32) staged candidates of token slot j in the row's list
      auto reserve = [&](int j, uint32_t n) {
        if (lane == 0) pbase[j] = atomicAdd(p.cnt + (it.t0 + col0 / H_I + j - p.row_begin) * p.state_ld, n);
        pend[j] = n;
        rcount[j] -= n;
      };
      // stores the reserved entries of token slot j (waits for the reservation's result)
      auto store_pending = [&](int j) {
        if (pend[j] == 0) return;
        const uint2* ring = reinterpret_cast<const uint2*>(smem + C::OFF_RING) + (ep * C::TPW + j) * C::RING;
        const long long rr = it.t0 + col0 / H_I + j - p.row_begin;
        const uint32_t base = __shfl_sync(0xffffffffu, pbase[j], 0);
        if ((uint32_t)lane < pend[j] && base + lane < (uint32_t)p.cap)
          p.cand[rr * p.cap + base + lane] = ring[(rhead[j] + lane) & (C::RING - 1)];
        rhead[j] = (rhead[j] + pend[j]) & (C::RING - 1);
        pend[j] = 0;
        __syncwarp();  // the ring slots just read may be refilled
      };
      for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
        if (!(ok = mbar_wait(&acc_full[ab], abph, abort_flag, 16))) break;
        tc_fence_after();
        const int s = tile * TILE_KEYS + (int)rank * 128 + lane_grp * 32 + lane;
        const uint32_t tbase = tmem_base + lane_off + ab * C::N + col0;
        float* out_row0 = p.scores + (it.t0 - p.row_begin) * p.ld + s;
#pragma unroll
        for (int c = 0; c < C::CPT; c += H_I) {
          const int tok = (col0 + c) / H_I;
          const int j = c / H_I;
          // four interleaved partial sums over the heads (h mod 4), added pairwise at the
          // end: a chain of H_I / 4 dependent FMAs instead of H_I
          float a4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int h0 = 0; h0 < H_I; h0 += 16) {
            float v[16];
            tmem_ld_x16_sync(tbase + c + h0, v);
#pragma unroll
            for (int q = 0; q < 16; q += 2) {
              const uint32_t pr = wp[(c + h0 + q) / 2];
              a4[q & 3] = fmaf(__uint_as_float(pr << 16), fmaxf(v[q], 0.f), a4[q & 3]);
              a4[(q + 1) & 3] = fmaf(__uint_as_float(pr & 0xFFFF0000u), fmaxf(v[q + 1], 0.f), a4[(q + 1) & 3]);
            }
          }
          const float acc = (a4[0] + a4[1]) + (a4[2] + a4[3]);
          if constexpr (!FUSED) {
            if (s < vtok[j]) out_row0[(long long)tok * p.ld] = acc;
          } else {
            // the ring holds at most 31 staged entries here (the reservation of the previous
            // visit is stored first), so 32 new ones never overrun its 64 slots
            store_pending(j);
            const uint32_t key = float_order_key(acc);
            const bool pass = s < vtok[j] && key >= thr_t[j];
            const uint32_t m = __ballot_sync(0xffffffffu, pass);
            if (m) {
              uint2* ring = reinterpret_cast<uint2*>(smem + C::OFF_RING) + (ep * C::TPW + j) * C::RING;
              if (pass)
                ring[(rhead[j] + rcount[j] + __popc(m & ((1u << lane) - 1u))) & (C::RING - 1)] =
                    make_uint2(key, (uint32_t)s);
              rcount[j] += __popc(m);
              __syncwarp();
              if (rcount[j] >= 32) reserve(j, 32);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(ab == 0 ? acc_empty0 : acc_empty1);
        if (++ab == 2) { ab = 0; abph ^= 1; }
      }
      if constexpr (FUSED) {
        if (ok) {
#pragma unroll
          for (int j = 0; j < C::TPW; ++j) {
            store_pending(j);
            if (rcount[j] > 0) {
              reserve(j, rcount[j]);
              store_pending(j);
            }
          }
        }
      }
      item = nitem;
      it = nx;
      have = have_next;
      wbuf ^= 1;
    }
    cp_async_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA of the pair leaves while the other may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc2(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

namespace dsa_host {

// Which form of the CTA-pair kernel a launch runs (see the kernel's header comment).
struct Indexer2Pass {
  int key_stride = 1;             // > 1: sampled scores over every key_stride-th key
  const int* mark = nullptr;      // repair: rows marked -2 in mark[(r - row_begin) * mark_ld]
  int mark_ld = 0;
  const int* run_flag = nullptr;  // repair: nothing to do while *run_flag == 0
  const uint32_t* thr = nullptr;  // fused: per-row bound and candidate count (row stride
  uint32_t* cnt = nullptr;        // state_ld) and candidate lists
  long long state_ld = 1;
  uint2* cand = nullptr;
  int cap = 0;
};

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES, bool FUSED>
static int launch_indexer2(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                           int batch, long long total_q, long long total_k, int max_seqlen_k, long long row_begin,
                           long long row_end, float* scores, long long ld, int tiles_per_split,
                           const Indexer2Pass& pass, cudaStream_t stream) {
  using C = dsa::Indexer2Cfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES, FUSED>;
  auto kern = dsa::indexer2_kernel<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES, FUSED>;
  static DeviceFlag attr_done;
  const int smem = std::max(C::SMEM_BYTES, 120 * 1024);
  if (!attr_done) {
    const cudaError_t e_ = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e_ != cudaSuccess) return cuda_fail(e_);
    // the register reallocation must fit what the launch holds, or its increase would wait
    // for registers that never come: check the compiled register count once
    cudaFuncAttributes fa;
    if (const cudaError_t e2 = cudaFuncGetAttributes(&fa, kern); e2 != cudaSuccess) return cuda_fail(e2);
    if ((long long)fa.numRegs * C::THREADS < 128LL * C::REG_ROLE + (long long)C::EPI_THREADS * C::REG_EPI)
      return DSA_ERR_UNSUPPORTED;
    attr_done = true;
  }
  const long long S = std::max(1, pass.key_stride);
  CUtensorMap tk, tq;
  // sampled scores: the key map steps S rows of k_idx per row (rows past the end read 0)
  int st = make_tmap_bf16_2d(&tk, k_idx, (uint64_t)((total_k + S - 1) / S), D_I, (uint64_t)(S * D_I * 2), 128,
                             C::PANEL, C::SWZ);
  if (st != DSA_OK) return st;
  st = make_tmap_bf16_2d(&tq, q_idx, (uint64_t)total_q * H_I, D_I, (uint64_t)D_I * 2, C::NH, C::PANEL, C::SWZ);
  if (st != DSA_OK) return st;
  dsa::IndexerParams p;
  p.w = static_cast<const uint16_t*>(w);
  p.w_elems = total_q * H_I;
  p.cu_q = cu_q;
  p.cu_k = cu_k;
  p.batch = batch;
  p.row_begin = row_begin;
  p.row_end = row_end;
  p.scores = scores;
  p.ld = ld;
  p.tiles_per_split = tiles_per_split;
  p.key_stride = (int)S;
  p.mark = pass.mark;
  p.mark_ld = pass.mark_ld;
  p.run_flag = pass.run_flag;
  p.thr = pass.thr;
  p.cnt = pass.cnt;
  p.state_ld = pass.state_ld;
  p.cand = pass.cand;
  p.cap = pass.cap;
  const long long max_keys = S == 1 ? max_seqlen_k : max_seqlen_k / S + 2;
  const long long max_tiles = (max_keys + 255) / 256;
  p.max_splits = (int)std::max(1LL, (max_tiles + tiles_per_split - 1) / tiles_per_split);
  const long long rows = row_end - row_begin;
  const long long nblk = (rows + NTOK - 1) / NTOK + batch;
  p.n_items = nblk * p.max_splits;
  const long long pairs = std::min<long long>(p.n_items, (long long)(sm_count() / 2));
  if (pairs <= 0) return DSA_OK;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (const cudaError_t e_ = cudaLaunchKernelEx(&cfg, kern, tk, tq, p); e_ != cudaSuccess) return cuda_fail(e_);
  return last_launch_status();
}

// True for the indexer shapes that have the CTA-pair kernel (and so the fused top-k).
bool indexer2_shape(int H_I, int d_I) { return d_I == 128 && (H_I == 64 || H_I == 32); }

// Any form of the CTA-pair kernel for the 128K-class prefill shapes; fused = candidates
// instead of scores.  DSA_ERR_UNSUPPORTED for other shapes.
int indexer2_pass_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                         int batch, long long total_q, long long total_k, int max_seqlen_k, int H_I, int d_I,
                         long long row_begin, long long row_end, float* scores, long long ld, bool fused,
                         const Indexer2Pass& pass, cudaStream_t stream) {
#define DSA_IDX2(HI, NT, FU)                                                                                  \
  return launch_indexer2<HI, 128, NT, 8, 4, 2, FU>(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k,      \
                                                   max_seqlen_k, row_begin, row_end, scores, ld, 64, pass, stream)
  if (H_I == 64 && d_I == 128) {
    if (fused) DSA_IDX2(64, 4, true);
    DSA_IDX2(64, 4, false);
  }
  if (H_I == 32 && d_I == 128) {
    if (fused) DSA_IDX2(32, 8, true);
    DSA_IDX2(32, 8, false);
  }
#undef DSA_IDX2
  return DSA_ERR_UNSUPPORTED;
}

// 128K-class prefill shapes on CTA pairs, scores form; DSA_ERR_UNSUPPORTED for other shapes
int indexer2_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                    long long total_q, long long total_k, int max_seqlen_k, int H_I, int d_I, long long row_begin,
                    long long row_end, float* scores, long long ld, cudaStream_t stream) {
  return indexer2_pass_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I,
                              row_begin, row_end, scores, ld, false, Indexer2Pass{}, stream);
}

}  // namespace dsa_host
