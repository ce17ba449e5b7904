// Lightning-indexer scores on tcgen05 tensor cores (sm_100a).
//
//   I[t,s] = sum_j w[t,j] * max(0, q_idx[t,j,:] . k_idx[s,:])        (s visible to t)
//
// Source: Keye-VL-2.0 report summary (mqxn.cn/news/1966), section 1: one lightweight,
// MQA-shared indexer scans every position for each query token.
//
// Design (swap-AB):  M = 128 keys per tile (A = k_idx rows, K-major),
//                    N = NTOK tokens x H_I heads (B = q_idx rows, K-major),
//                    K = d_I.
// Each TMEM lane then holds one key and each column one (token, head), so the ReLU, the
// w-weighting and the sum over heads are thread-local in the epilogue.  The CTA is
// persistent and warp-specialised:
//   warp 0      TMA producer: q_idx block once per work item, k_idx tiles in a ring
//   warp 1      MMA issuer (one thread) + TMEM owner; two accumulator buffers in TMEM
//   warps 2..   epilogue: tcgen05.ld -> fp32 ReLU/FMA over heads -> coalesced stores
// A work item is (token block of NTOK rows of one sequence, a range of key tiles); items
// are visited heaviest-first so the causal triangle balances across SMs.
#include <algorithm>
#include <cstdio>

#include "common.cuh"

namespace dsa {

struct IndexerParams {
  const uint16_t* w;  // [total_q, H_I] bf16
  long long w_elems;  // total_q * H_I
  const int* cu_q;
  const int* cu_k;
  int batch;
  long long row_begin, row_end;
  float* scores;
  long long ld;
  int tiles_per_split;
  int max_splits;
  long long n_items;
  // Sampled scores: with key_stride S > 1 the keys are the k_idx rows 0, S, 2S, ... (the
  // key tensor map steps S rows at a time) and score column j of a row is the key at
  // packed row (ceil(k0 / S) + j) * S, for the visible ones.
  int key_stride = 1;
  // Repair pass: only blocks holding a row r with mark[(r - row_begin) * mark_ld] == -2
  // are processed, and nothing at all while *run_flag == 0.
  const int* mark = nullptr;
  int mark_ld = 0;
  const int* run_flag = nullptr;
  // Fused top-k candidates (CTA-pair kernel, fused form): scores whose order key is at
  // least thr[(r - row_begin) * state_ld] are appended as (key, position) to
  // cand[(r - row_begin) * cap ..] with the running count in cnt[(r - row_begin) * state_ld];
  // no score matrix is written.
  const uint32_t* thr = nullptr;
  uint32_t* cnt = nullptr;
  long long state_ld = 1;
  uint2* cand = nullptr;
  int cap = 0;
};

struct Item {
  long long t0;  // first packed query row of the block
  int ntok;      // valid rows in the block
  int i0;        // sequence-local index of row t0
  int Lq, Lk;
  int kg;        // first packed key row of the sequence
  int k0;        // first key-tensor-map row of the sequence (kg, or ceil(kg / S) when sampled)
  int tile_begin, tile_end;
};

// Visible keys of a row in the key-tensor-map rows of the item: the causal count, or for
// sampled scores the number of sampled rows j * S inside [kg, kg + vis).
__device__ __forceinline__ int item_visible(const IndexerParams& p, const Item& it, int vis) {
  if (p.key_stride == 1) return vis;
  const long long S = p.key_stride;
  return (int)((it.kg + (long long)vis + S - 1) / S - it.k0);
}

// Work item -> (token block, key-tile range).  Items are numbered split-major
// (item = split * blocks + block) with blocks heaviest-first, so consecutive item numbers,
// which go to consecutive CTAs, are all non-empty for the first split of every block and
// the empty (split beyond a light block's tiles) items bunch up at the end.
template <int NTOK, int TILE_KEYS = 128>
__device__ __forceinline__ bool decode_item(long long item, const IndexerParams& p, Item& it) {
  // count the blocks in this row chunk; blocks are numbered from the last one (heaviest)
  long long total = 0;
  for (int b = 0; b < p.batch; ++b) {
    const long long lo = max((long long)p.cu_q[b], p.row_begin);
    const long long hi = min((long long)p.cu_q[b + 1], p.row_end);
    if (hi > lo) total += (hi - lo + NTOK - 1) / NTOK;
  }
  if (total == 0) return false;
  const long long split_ll = item / total;
  if (split_ll >= p.max_splits) return false;
  const int split = (int)split_ll;
  const long long blk = item % total;
  long long r = total - 1 - blk;  // ascending block number
  for (int b = 0; b < p.batch; ++b) {
    const long long lo = max((long long)p.cu_q[b], p.row_begin);
    const long long hi = min((long long)p.cu_q[b + 1], p.row_end);
    if (hi <= lo) continue;
    const long long nb = (hi - lo + NTOK - 1) / NTOK;
    if (r < nb) {
      it.t0 = lo + r * NTOK;
      it.ntok = (int)min((long long)NTOK, hi - it.t0);
      it.i0 = (int)(it.t0 - p.cu_q[b]);
      it.Lq = p.cu_q[b + 1] - p.cu_q[b];
      it.Lk = p.cu_k[b + 1] - p.cu_k[b];
      it.kg = p.cu_k[b];
      it.k0 = p.key_stride == 1 ? it.kg : (int)(((long long)it.kg + p.key_stride - 1) / p.key_stride);
      const int last = it.i0 + it.ntok - 1;
      const int vis = item_visible(p, it, min(max(last + it.Lk - it.Lq + 1, 0), it.Lk));
      const int ntiles = (vis + TILE_KEYS - 1) / TILE_KEYS;
      it.tile_begin = split * p.tiles_per_split;
      it.tile_end = min(ntiles, it.tile_begin + p.tiles_per_split);
      if (it.tile_begin >= it.tile_end) return false;
      if (p.mark) {
        bool any = false;
        for (int j = 0; j < it.ntok; ++j) any |= p.mark[(it.t0 + j - p.row_begin) * p.mark_ld] == -2;
        return any;
      }
      return true;
    }
    r -= nb;
  }
  return false;
}

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES>
struct IndexerCfg {
  static constexpr int N = NTOK * H_I;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "UMMA N");
  static constexpr int PANEL = D_I >= 64 ? 64 : D_I;  // elements per swizzle row
  static constexpr int SWZ = PANEL * 2;               // 128 or 64 bytes
  static constexpr int NPANEL = D_I / PANEL;
  static constexpr int KSTEPS = PANEL / 16;
  static constexpr int A_BYTES = 128 * D_I * 2;
  static constexpr int B_BYTES = N * D_I * 2;
  static constexpr int TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr int EPI_THREADS = NUM_EPI_WARPS * 32;
  static constexpr int THREADS = 64 + EPI_THREADS;
  static constexpr int COL_PARTS = NUM_EPI_WARPS / 4;
  static constexpr int CPT = N / COL_PARTS;  // accumulator columns per epilogue thread
  static_assert(CPT % 32 == 0, "epilogue reads 32-column chunks");
  // shared memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + A_STAGES * A_BYTES;
  static constexpr int OFF_W = OFF_B + B_STAGES * B_BYTES;
  static constexpr int OFF_BAR = OFF_W + N * 4;
  static constexpr int NUM_BARS = 2 * A_STAGES + 2 * B_STAGES + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
  static constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;  // + alignment slack
  static constexpr uint32_t IDESC = idesc_bf16_f32(128, N);
  static_assert(SMEM_BYTES <= 232448, "exceeds the 227 KB per-block shared memory limit");
};

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES>
__global__ void __launch_bounds__(IndexerCfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES>::THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                   const IndexerParams p) {
  using C = IndexerCfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES>;
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::OFF_A;
  uint8_t* sB = smem + C::OFF_B;
  float* sW = reinterpret_cast<float*>(smem + C::OFF_W);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* a_full = bars;
  uint64_t* a_empty = bars + A_STAGES;
  uint64_t* b_full = bars + 2 * A_STAGES;
  uint64_t* b_empty = bars + 2 * A_STAGES + B_STAGES;
  uint64_t* acc_full = bars + 2 * A_STAGES + 2 * B_STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* mma_done = acc_full + 4;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 8);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

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
      mbar_init(&acc_empty[i], NUM_EPI_WARPS);
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
      int as = 0, bs = 0;
      uint32_t aph = 0, bph = 0;
      bool ok = true;
      for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        Item it;
        if (!decode_item<NTOK>(item, p, it)) continue;
        if (!(ok = mbar_wait(&b_empty[bs], bph ^ 1, abort_flag, 1))) break;
        mbar_arrive_expect_tx(&b_full[bs], C::B_BYTES);
        for (int pn = 0; pn < C::NPANEL; ++pn)
          tma_load_2d(sB + bs * C::B_BYTES + pn * C::N * C::SWZ, &tmap_q, &b_full[bs], pn * C::PANEL,
                      (int)(it.t0 * H_I));
        if (++bs == B_STAGES) { bs = 0; bph ^= 1; }
        for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
          if (!(ok = mbar_wait(&a_empty[as], aph ^ 1, abort_flag, 2))) break;
          mbar_arrive_expect_tx(&a_full[as], C::A_BYTES);
          for (int pn = 0; pn < C::NPANEL; ++pn)
            tma_load_2d(sA + as * C::A_BYTES + pn * 128 * C::SWZ, &tmap_k, &a_full[as], pn * C::PANEL,
                        it.k0 + tile * 128);
          if (++as == A_STAGES) { as = 0; aph ^= 1; }
        }
      }
      if (!ok) {
        // drain: let every load this thread issued land before the CTA can exit
        for (int i = 0; i < A_STAGES; ++i) {
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(smem_u32(&a_full[i]), aph ^ (i >= as ? 1u : 0u)) &&
                 globaltimer_ns() - t0 < 200000000ull) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int as = 0, bs = 0, ab = 0;
      uint32_t aph = 0, bph = 0, abph = 0;
      bool ok = true;
      for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
        Item it;
        if (!decode_item<NTOK>(item, p, it)) continue;
        if (!(ok = mbar_wait(&b_full[bs], bph, abort_flag, 3))) break;
        const uint32_t b_base = smem_u32(sB + bs * C::B_BYTES);
        for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
          if (!(ok = mbar_wait(&acc_empty[ab], abph ^ 1, abort_flag, 4))) break;
          tc_fence_after();
          if (!(ok = mbar_wait(&a_full[as], aph, abort_flag, 5))) break;
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + as * C::A_BYTES);
          const uint32_t d_tmem = tmem_base + ab * C::N;
#pragma unroll
          for (int pn = 0; pn < C::NPANEL; ++pn) {
#pragma unroll
            for (int kk = 0; kk < C::KSTEPS; ++kk) {
              const uint64_t adesc = smem_desc_kmajor(a_base + pn * 128 * C::SWZ + kk * 32, C::SWZ);
              const uint64_t bdesc = smem_desc_kmajor(b_base + pn * C::N * C::SWZ + kk * 32, C::SWZ);
              umma_bf16(d_tmem, adesc, bdesc, C::IDESC, (pn | kk) != 0);
            }
          }
          umma_commit(&a_empty[as]);
          umma_commit(&acc_full[ab]);
          if (++as == A_STAGES) { as = 0; aph ^= 1; }
          if (++ab == 2) { ab = 0; abph ^= 1; }
        }
        if (!ok) break;
        umma_commit(&b_empty[bs]);
        if (++bs == B_STAGES) { bs = 0; bph ^= 1; }
      }
      // wait for every MMA this thread issued before TMEM can be released
      umma_commit(mma_done);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(smem_u32(mma_done), 0) && globaltimer_ns() - t0 < 200000000ull) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ep = warp - 2;               // 0 .. NUM_EPI_WARPS-1
    const int lane_grp = warp % 4;         // TMEM lane quarter this warp may access
    const int col_part = ep / 4;           // which share of the N columns
    const int ep_tid = ep * 32 + lane;
    const int col0 = col_part * C::CPT;
    const uint32_t lane_off = (uint32_t)(lane_grp * 32) << 16;
    int ab = 0;
    uint32_t abph = 0;
    bool ok = true;
    float* w_s = sW;
    for (long long item = blockIdx.x; item < p.n_items && ok; item += gridDim.x) {
      Item it;
      if (!decode_item<NTOK>(item, p, it)) continue;
      named_bar_sync(1, C::EPI_THREADS);  // every epilogue thread is done with the previous weights
      for (int i = ep_tid; i < C::N; i += C::EPI_THREADS) {
        const int t = i / H_I;
        w_s[i] = (t < it.ntok) ? bf16_bits_to_f32(p.w[(it.t0 + t) * H_I + (i % H_I)]) : 0.f;
      }
      named_bar_sync(1, C::EPI_THREADS);
      const int dvis = it.Lk - it.Lq + 1;  // vis(i) = clamp(i + dvis, 0, Lk)
      // this thread's weights for the whole item (reused by every key tile): keeping them in
      // registers leaves the shared-memory pipe to the tensor core's operand reads
      float wr[H_I >= 32 ? C::CPT : 1];
      if constexpr (H_I >= 32) {
#pragma unroll
        for (int c = 0; c < C::CPT; ++c) wr[c] = w_s[col0 + c];
      }
      for (int tile = it.tile_begin; tile < it.tile_end; ++tile) {
        if (!(ok = mbar_wait(&acc_full[ab], abph, abort_flag, 6))) break;
        tc_fence_after();
        const int s = tile * 128 + lane_grp * 32 + lane;  // this thread's key (sequence-local)
        const uint32_t tbase = tmem_base + lane_off + ab * C::N + col0;
        float* out_row0 = p.scores + (it.t0 - p.row_begin) * p.ld + s;
        if constexpr (H_I >= 32) {
#pragma unroll
          for (int c = 0; c < C::CPT; c += H_I) {
            const int tok = (col0 + c) / H_I;
            float acc = 0.f;
#pragma unroll
            for (int h0 = 0; h0 < H_I; h0 += 16) {
              float v[16];
              tmem_ld_x16_sync(tbase + c + h0, v);
#pragma unroll
              for (int q = 0; q < 16; ++q) acc = fmaf(wr[c + h0 + q], fmaxf(v[q], 0.f), acc);
            }
            const int vis = min(max(it.i0 + tok + dvis, 0), it.Lk);
            if (tok < it.ntok && s < vis) out_row0[(long long)tok * p.ld] = acc;
          }
        } else {
          constexpr int TPC = 32 / H_I;  // tokens per 32-column chunk
#pragma unroll 1
          for (int c = 0; c < C::CPT; c += 32) {
            float v[32];
            tmem_ld_x32_sync(tbase + c, v);
            const int tok_base = (col0 + c) / H_I;
#pragma unroll
            for (int u = 0; u < TPC; ++u) {
              const int tok = tok_base + u;
              float acc = 0.f;
#pragma unroll
              for (int h = 0; h < H_I; ++h) acc = fmaf(w_s[tok * H_I + h], fmaxf(v[u * H_I + h], 0.f), acc);
              const int vis = min(max(it.i0 + tok + dvis, 0), it.Lk);
              if (tok < it.ntok && s < vis) out_row0[(long long)tok * p.ld] = acc;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[ab]);
        if (++ab == 2) { ab = 0; abph ^= 1; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace dsa

// ====================================================================== host launcher
namespace dsa_host {

template <int H_I, int D_I, int NTOK, int NUM_EPI_WARPS, int A_STAGES, int B_STAGES>
static int launch_indexer(const void* q_idx, const void* k_idx, const void* w, const int* cu_q,
                          const int* cu_k, int batch, long long total_q, long long total_k,
                          int max_seqlen_q, int max_seqlen_k, long long row_begin, long long row_end,
                          float* scores, long long ld, int tiles_per_split, cudaStream_t stream) {
  using C = dsa::IndexerCfg<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES>;
  auto kern = dsa::indexer_kernel<H_I, D_I, NTOK, NUM_EPI_WARPS, A_STAGES, B_STAGES>;
  static DeviceFlag attr_done;
  const int smem = std::max(C::SMEM_BYTES, 120 * 1024);  // one CTA per SM (TMEM ownership)
  if (!attr_done) {
    if (const cudaError_t e_ = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); e_ != cudaSuccess) return cuda_fail(e_);
    attr_done = true;
  }
  CUtensorMap tk, tq;
  int st = make_tmap_bf16_2d(&tk, k_idx, (uint64_t)total_k, D_I, (uint64_t)D_I * 2, 128, C::PANEL, C::SWZ);
  if (st != DSA_OK) return st;
  st = make_tmap_bf16_2d(&tq, q_idx, (uint64_t)total_q * H_I, D_I, (uint64_t)D_I * 2, C::N, C::PANEL, C::SWZ);
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
  const int max_tiles = (max_seqlen_k + 127) / 128;
  p.max_splits = std::max(1, (max_tiles + tiles_per_split - 1) / tiles_per_split);
  const long long rows = row_end - row_begin;
  const long long nblk = (rows + NTOK - 1) / NTOK + batch;
  p.n_items = nblk * p.max_splits;
  (void)max_seqlen_q;
  const long long grid = std::min<long long>(p.n_items, (long long)sm_count());
  if (grid <= 0) return DSA_OK;
  return launch_pdl(false, kern, dim3((unsigned)grid), dim3(C::THREADS), (size_t)smem, stream, tk, tq, p);
}

int indexer2_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k, int batch,
                    long long total_q, long long total_k, int max_seqlen_k, int H_I, int d_I, long long row_begin,
                    long long row_end, float* scores, long long ld, cudaStream_t stream);

int indexer_launch(const void* q_idx, const void* k_idx, const void* w, const int* cu_q, const int* cu_k,
                   int batch, long long total_q, long long total_k, int max_seqlen_q, int max_seqlen_k,
                   int H_I, int d_I, long long row_begin, long long row_end, float* scores, long long ld,
                   cudaStream_t stream) {
  const long long rows = row_end - row_begin;
  // Few query rows per sequence (decode): one token per block, split the keys finely.
  const bool decode_like = rows <= 2LL * batch;
  // Many rows: CTA pairs (tcgen05 cta_group::2) for the 128-wide indexer heads.
  if (!decode_like && d_I == 128 && (H_I == 64 || H_I == 32))
    return indexer2_launch(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k, max_seqlen_k, H_I, d_I, row_begin,
                           row_end, scores, ld, stream);
#define DSA_IDX(HI, DI, NT, EW, AS, BS, TPS)                                                                  \
  return launch_indexer<HI, DI, NT, EW, AS, BS>(q_idx, k_idx, w, cu_q, cu_k, batch, total_q, total_k,     \
                                                max_seqlen_q, max_seqlen_k, row_begin, row_end, scores, ld, \
                                                TPS, stream)
  if (H_I == 64 && d_I == 128) {
    if (decode_like) DSA_IDX(64, 128, 1, 4, 6, 2, 16);
    DSA_IDX(64, 128, 4, 8, 3, 2, 64);
  }
  if (H_I == 32 && d_I == 128) {
    if (decode_like) DSA_IDX(32, 128, 2, 4, 6, 2, 16);
    DSA_IDX(32, 128, 8, 8, 3, 2, 64);
  }
  if (H_I == 16 && d_I == 128) DSA_IDX(16, 128, 16, 8, 3, 2, 64);
  if (H_I == 8 && d_I == 64) DSA_IDX(8, 64, 32, 8, 4, 2, 64);
  if (H_I == 4 && d_I == 32) DSA_IDX(4, 32, 64, 8, 6, 2, 64);
#undef DSA_IDX
  return DSA_ERR_UNSUPPORTED;
}

}  // namespace dsa_host
