// bf16 Sep-Attention prefill on tcgen05 tensor cores (sm_100a).
//
// What it computes ("HKUDS047: SepLLM ..." study, section "SepAttention";
// jieyibu.net explainer, section 1.2): for query row i,
//   out_i = sum_{j in K_i} softmax(scale * q_i . k_j) v_j,
//   K_i = { j <= i : j < a  or  is_sep[j]  or  i - j < n }.
//
// Key sets of a 128-row tile [q0, q0+128), with lo = max(0, q0 - n + 1):
//   * the gathered set -- initial tokens [0, min(a, lo)) and separators in
//     [a, lo).  Every row of the tile keeps all of them, so their blocks need
//     no element mask.  A small kernel first copies, per (b, kv head), the
//     K/V rows of the initial tokens followed by every separator at a
//     position >= a into a contiguous workspace buffer; the gathered set of
//     any tile is then a prefix of that list, loaded with plain TMA tiles.
//   * the window range [lo, q0 + 128), loaded contiguously from K/V, with the
//     element mask  j >= lo, j <= i and (i - j < n or is_sep[j] or j < a).
// Each key of K_i is scored exactly once.
//
// Work item = two 128-row tiles that share one key stream:
//   * GQA (an even number of query heads per kv head): the same rows of two
//     query heads of one group -- identical key sets;
//   * otherwise: rows [q0, q0+128) and [q0+128, q0+256) of one head -- the
//     stream is the union (the larger gathered prefix and the window range
//     from the first tile's lo); per-tile masks keep each tile's own set.
// The kernel is persistent (one CTA per SM); items are numbered heaviest
// first and handed out dynamically (a global counter read by the producer,
// passed to the other roles through a shared-memory ring, see publish_item).
// Warps 0-3 and 4-7 are the softmax warpgroups of tiles A
// and B (thread = query row = TMEM lane), warp 8 issues TMA loads, warps 9
// and 10 issue the tcgen05.mma of tiles A and B (warp 9 owns TMEM).  TMEM:
// S_A | S_B | O_A | O_B, and for D = 64 also P_A | P_B, so that S of the next
// block is computed while the softmax of this one still runs; for D = 128 a
// tile's P (bf16) is written over the first 64 columns of its S.  P feeds
// the PV MMA from TMEM.  While one warpgroup runs its softmax the tensor
// core works on the other tile, and the next item's Q/K/V loads overlap the
// current item's tail.  The reference maximum moves (and O is rescaled) only
// when a block's row sum would exceed 2^16, and then to the block's exact
// maximum.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per block
constexpr int kThreads = 352;
constexpr int kTmaWarp = 8;
constexpr int kMmaWarp = 9;   // MMA issuer of tile A (and TMEM owner)
constexpr int kMmaWarpB = 10; // MMA issuer of tile B
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Cfg {
  static constexpr int NST = D == 64 ? 4 : 2;  // K/V shared-memory stages
  static constexpr int REG = 128 * 128;        // one 64-column region of a 128-row tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_QA = 0;
  static constexpr int OFF_QB = OFF_QA + Q_BYTES;
  static constexpr int OFF_K = OFF_QB + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NST * KV_BYTES;
  // D = 64: per-tile staging of the output tile for one tensor store
  static constexpr int OFF_STG = OFF_V + NST * KV_BYTES;
  static constexpr int STG_BYTES = D == 64 ? 2 * Q_BYTES : 0;
  static constexpr int OFF_BAR = OFF_STG + STG_BYTES;
  static constexpr int BYTES = OFF_BAR + 512;
  static constexpr int ALLOC = BYTES + 1024;  // slack for 1024-byte alignment
  static constexpr uint32_t COL_S0 = 0, COL_S1 = 128, COL_O0 = 256, COL_O1 = 256 + D;
  // D = 64 leaves room for a separate P region per tile (bf16 pairs of 128
  // keys in 64 columns): S of the next block can then be computed while the
  // softmax of this one is still running.  D = 128 writes P over S.
  static constexpr bool SEP_P = D == 64;
  static constexpr uint32_t COL_P0 = SEP_P ? 384 : COL_S0, COL_P1 = SEP_P ? 448 : COL_S1;
};

template <int NST>
struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t s_free[2], pv_done[2];  // separate-P protocol: S read back / P*V done
  uint64_t drain;
  uint64_t it_full[4], it_empty[4];  // work-item ring (dynamic scheduling)
  int item_q[4];
  uint32_t tmem_base;
  int abort;
};

struct Params {
  const uint8_t* is_sep;
  const int32_t* prefix;
  int B, Hq, Hkv, S, a, n, G;
  int pair_heads;  // 1: the two tiles are two heads of a group; 0: two row tiles of one head
  int npairs, ntiles_item, n_items;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  int32_t* err;
  int32_t* sched;  // next work item (zeroed by the gather kernel before each launch)
};

// Geometry of one work item, computed identically by every role.
struct Item {
  int b, g;
  int h[2];    // query head of tile A / B
  int q0[2];   // first row of tile A / B
  int lo[2];   // window start of tile A / B
  int nG[2];   // gathered keys of tile A / B (a prefix of the compact list)
  int win_lo;  // window range streamed: [win_lo, win_hi)
  int win_hi;
  int nblk_g, nblk;
};

__device__ __forceinline__ Item make_item(const Params& p, int item) {
  Item it;
  const int per_tile = p.B * p.npairs;
  const int qt = p.ntiles_item - 1 - item / per_tile;  // heaviest (last) tiles first
  const int rem = item % per_tile;
  it.b = rem / p.npairs;
  const int pr = rem % p.npairs;
  if (p.pair_heads) {
    it.h[0] = 2 * pr;
    it.h[1] = 2 * pr + 1;
    it.q0[0] = it.q0[1] = qt * BM;
  } else {
    it.h[0] = it.h[1] = pr;
    it.q0[0] = qt * 2 * BM;
    it.q0[1] = qt * 2 * BM + BM;
  }
  it.g = it.h[0] / p.G;
  const int32_t* pre = p.prefix + static_cast<int64_t>(it.b) * (p.S + 1);
  const int aa = p.a < p.S ? p.a : p.S;
  for (int t = 0; t < 2; ++t) {
    const int q0 = it.q0[t] < p.S ? it.q0[t] : p.S - 1;
    const int lo = q0 - p.n + 1 > 0 ? q0 - p.n + 1 : 0;
    it.lo[t] = lo;
    it.nG[t] = (p.a < lo ? p.a : lo) + (lo > aa ? pre[lo] - pre[aa] : 0);
  }
  const int nG_all = it.nG[0] > it.nG[1] ? it.nG[0] : it.nG[1];
  it.win_lo = it.lo[0] < it.lo[1] ? it.lo[0] : it.lo[1];
  const int hi = (it.q0[0] > it.q0[1] ? it.q0[0] : it.q0[1]) + BM;
  it.win_hi = hi < p.S ? hi : p.S;
  it.nblk_g = (nG_all + BN - 1) / BN;
  it.nblk = it.nblk_g + (it.win_hi - it.win_lo + BN - 1) / BN;
  return it;
}

// Does tile t keep any key of block j of its item's stream?  Gathered block
// j: j*128 < nG_t.  Window block at `base`: [base, base+128) meets
// [lo_t, last row of the tile] (keys below lo_t are the tile's gathered
// keys; keys above its last row are causal-masked).  Blocks no tile keeps
// are not streamed, and a tile skips the blocks it does not keep.
__device__ __forceinline__ bool block_active(const Item& it, int t, int j, int S) {
  if (j < it.nblk_g) return j * BN < (t ? it.nG[1] : it.nG[0]);
  const int base = it.win_lo + (j - it.nblk_g) * BN;
  const int q0 = t ? it.q0[1] : it.q0[0];
  const int last = q0 + BM - 1 < S - 1 ? q0 + BM - 1 : S - 1;
  const int lo = t ? it.lo[1] : it.lo[0];
  return base <= last && base + BN - 1 >= lo;
}

// mask of bit positions c in [0, 32) with c <= x
__device__ __forceinline__ uint32_t bits_le(int x) {
  return x < 0 ? 0u : (x >= 31 ? 0xffffffffu : (0xffffffffu >> (31 - x)));
}

// mbarrier phase wait: one (potentially blocking) try inline, the bounded
// retry loop out of line.  Inlined at each of the kernel's wait sites the
// loop costs some 9 KB of instructions; one shared copy keeps the code that
// the warps run per item small enough for the instruction cache.
__device__ __noinline__ bool mbar_wait_loop(uint64_t* bar, uint32_t parity, volatile int* abort,
                                            int32_t* err_word) {
  return sep::mbar_wait(bar, parity, abort, err_word);
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* err_word) {
  return sep::mbar_try_wait(bar, parity) || mbar_wait_loop(bar, parity, abort, err_word);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, nullptr);
}

// Dynamic work distribution.  The producer thread takes item indices from a
// global counter (the index order is heaviest first, so each CTA takes the
// heaviest item left when it is ready for one) and publishes its k-th item
// in slot k % 4 of a ring; the MMA issuers and the softmax warps take the
// items from the ring in the same order.  An index >= n_items ends the loop;
// -1 means the CTA is aborting.
template <int NST>
__device__ __forceinline__ int publish_item(Bars<NST>* bars, uint32_t k, const Params& p,
                                            volatile int* abort) {
  const uint32_t slot = k & 3u;
  if (k >= 4 && !mbar_wait(&bars->it_empty[slot], ((k >> 2) - 1) & 1, abort, p.err)) return -1;
  int item = atomicAdd(p.sched, 1);
  if (item > p.n_items) item = p.n_items;
  bars->item_q[slot] = item;
  sep::mbar_arrive(&bars->it_full[slot]);  // release: the slot's value is visible to the takers
  return item;
}

// whole_warp: all 32 lanes take the item and lane 0 frees the slot for them.
template <int NST>
__device__ __forceinline__ int take_item(Bars<NST>* bars, uint32_t k, const Params& p,
                                         volatile int* abort, bool whole_warp) {
  const uint32_t slot = k & 3u;
  const bool got = mbar_wait(&bars->it_full[slot], (k >> 2) & 1, abort, p.err);
  if (whole_warp ? !__all_sync(0xffffffffu, got) : !got) return -1;
  const int item = *reinterpret_cast<volatile int*>(&bars->item_q[slot]);
  if (whole_warp) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) sep::mbar_arrive(&bars->it_empty[slot]);
  } else {
    sep::mbar_arrive(&bars->it_empty[slot]);
  }
  return item;
}

// MMA issue for both tiles from one thread, P written over S (D = 128): per
// block, tile A's P*V of the previous block then its S, then tile B's.
template <int D>
__device__ __forceinline__ void mma_single_issuer(const Params& p, uint8_t* smem, uint32_t tmem,
                                                  Bars<Cfg<D>::NST>* bars, volatile int* abort) {
  using C = Cfg<D>;
  constexpr int NST = C::NST;
  constexpr uint32_t idesc_s = sep::idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t idesc_o = sep::idesc_bf16_f32(BM, D, true);
  // descriptors built once (see the per-tile issuers)
  const uint64_t dq0 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_QA), 16);
  const uint64_t dq1 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_QB), 16);
  const uint64_t dk0 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_K), 16);
  const uint64_t dv0 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_V), C::REG);
  uint32_t gblk = 0, nitem = 0, pphase = 0;  // bit t: phase of p_full[t]
  bool ok = true;
  bool v_ready = false;  // V of the block whose PVs are being issued has landed
  auto issue_pv = [&](int t, uint32_t vblk, bool first) -> bool {
    if (!mbar_wait(&bars->p_full[t], (pphase >> t) & 1u, abort, p.err)) return false;
    pphase ^= 1u << t;
    if (!v_ready && !mbar_wait(&bars->v_full[vblk % NST], (vblk / NST) & 1, abort, p.err))
      return false;
    v_ready = true;
    if (first && nitem > 0 && !mbar_wait(&bars->o_empty[t], (nitem - 1) & 1, abort, p.err))
      return false;
    sep::tc_fence_after();
    const uint64_t dv = dv0 + static_cast<uint64_t>((vblk % NST) * (C::KV_BYTES >> 4));
    const uint32_t ptm = tmem + (t ? C::COL_P1 : C::COL_P0);
    const uint32_t otm = tmem + (t ? C::COL_O1 : C::COL_O0);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk)
      sep::mma_bf16_ts(otm, ptm + kk * 8, dv + kk * (2048 >> 4), idesc_o, (!first || kk > 0) ? 1u : 0u);
    return true;
  };
  auto issue_s = [&](int t, uint32_t kblk) {
    const uint64_t dk = dk0 + static_cast<uint64_t>((kblk % NST) * (C::KV_BYTES >> 4));
    const uint64_t dq = t ? dq1 : dq0;
    const uint32_t stm = tmem + (t ? C::COL_S1 : C::COL_S0);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::REG + (kk % 4) * 32) >> 4);
      sep::mma_bf16_ss(stm, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
    }
    sep::mma_commit(&bars->s_full[t]);
  };
  for (; ok; ++nitem) {
    const int item = take_item<NST>(bars, nitem, p, abort, false);
    if (item < 0 || item >= p.n_items) break;
    const Item it = make_item(p, item);
    if (!mbar_wait(&bars->q_full, nitem & 1, abort, p.err)) break;
    bool prev_a = false, prev_b = false;  // tile kept the previous block
    bool pv_a = false, pv_b = false;      // tile already accumulated into O this item
    for (int j = 0; j < it.nblk; ++j, ++gblk) {
      if (!mbar_wait(&bars->k_full[gblk % NST], (gblk / NST) & 1, abort, p.err)) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      const bool act_a = block_active(it, 0, j, p.S), act_b = block_active(it, 1, j, p.S);
      v_ready = false;
      if (prev_a) {
        if (!(ok = issue_pv(0, gblk - 1, !pv_a))) break;
        pv_a = true;
      }
      if (act_a) issue_s(0, gblk);
      if (prev_b) {
        if (!(ok = issue_pv(1, gblk - 1, !pv_b))) break;
        pv_b = true;
      }
      if (j > 0) sep::mma_commit(&bars->v_empty[(gblk - 1) % NST]);
      if (act_b) issue_s(1, gblk);
      sep::mma_commit(&bars->k_empty[gblk % NST]);
      if (j == it.nblk - 1) sep::mma_commit(&bars->q_empty);
      prev_a = act_a;
      prev_b = act_b;
    }
    if (!ok) break;
    // last block's P*V of both tiles, then hand O to the epilogues
    v_ready = false;
    if (prev_a && !(ok = issue_pv(0, gblk - 1, !pv_a))) break;
    sep::mma_commit(&bars->o_full[0]);
    if (prev_b && !(ok = issue_pv(1, gblk - 1, !pv_b))) break;
    sep::mma_commit(&bars->o_full[1]);
    sep::mma_commit(&bars->v_empty[(gblk - 1) % NST]);
  }
  sep::mma_commit(&bars->drain);
  drain_wait(&bars->drain, 0);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_prefill_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const __grid_constant__ CUtensorMap tm_o,
                 const Params p) {
  using C = Cfg<D>;
  constexpr int NST = C::NST;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Bars<NST>* bars = reinterpret_cast<Bars<NST>*>(smem + C::OFF_BAR);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    sep::mbar_init(&bars->q_full, 1);
    constexpr uint32_t kIssuers = C::SEP_P ? 2 : 1;  // one commit per MMA issuer
    sep::mbar_init(&bars->q_empty, kIssuers);
    for (int s = 0; s < NST; ++s) {
      sep::mbar_init(&bars->k_full[s], 1);
      sep::mbar_init(&bars->k_empty[s], kIssuers);
      sep::mbar_init(&bars->v_full[s], 1);
      sep::mbar_init(&bars->v_empty[s], kIssuers);
    }
    for (int t = 0; t < 2; ++t) {
      sep::mbar_init(&bars->s_full[t], 1);
      sep::mbar_init(&bars->p_full[t], 128);
      sep::mbar_init(&bars->o_full[t], 1);
      sep::mbar_init(&bars->o_empty[t], 128);
      sep::mbar_init(&bars->s_free[t], 128);
      sep::mbar_init(&bars->pv_done[t], 1);
    }
    sep::mbar_init(&bars->drain, kIssuers);
    for (int k = 0; k < 4; ++k) {
      sep::mbar_init(&bars->it_full[k], 1);
      sep::mbar_init(&bars->it_empty[k], kIssuers + 8);  // issuers + softmax warps
    }
    bars->abort = 0;
    sep::mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    sep::tmem_alloc(&bars->tmem_base, kTmemCols);
    sep::tmem_relinquish();
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // launched with programmatic serialization: the set-up above overlapped
  // the previous kernel; its outputs (index, gathered rows) are read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      sep::tma_prefetch_desc(&tm_q);
      sep::tma_prefetch_desc(&tm_k);
      sep::tma_prefetch_desc(&tm_v);
      sep::tma_prefetch_desc(&tm_kc);
      sep::tma_prefetch_desc(&tm_vc);
      // L2 policies: a Q tile is read once; the compact initial+separator
      // rows of a (b, kv head) are read by every later tile of it, so they
      // are kept over the streams of Q and of the outputs
      const uint64_t pol_q = sep::l2_evict_first_policy();
      const uint64_t pol_g = sep::l2_evict_last_policy();
      uint32_t gblk = 0, nitem = 0;
      int last_k[NST], last_v[NST];
      for (int s2 = 0; s2 < NST; ++s2) last_k[s2] = last_v[s2] = -1;
      int last_q = -1;
      bool ok = true;
      for (; ok; ++nitem) {
        const int item = publish_item<NST>(bars, nitem, p, abort);
        if (item < 0 || item >= p.n_items) break;
        const Item it = make_item(p, item);
        const int64_t kv_row0 = static_cast<int64_t>(it.b * p.Hkv + it.g) * p.S;
        if (nitem > 0 && !mbar_wait(&bars->q_empty, (nitem - 1) & 1, abort, p.err)) break;
        sep::mbar_arrive_expect_tx(&bars->q_full, 2 * C::Q_BYTES);
        for (int t = 0; t < 2; ++t) {
          const int64_t qrow = static_cast<int64_t>(it.b * p.Hq + it.h[t]) * p.S + it.q0[t];
          uint8_t* dst = smem + (t ? C::OFF_QB : C::OFF_QA);
#pragma unroll
          for (int r = 0; r < D / 64; ++r)
            sep::tma_load_2d_hint(dst + r * C::REG, &tm_q, r * 64, static_cast<int32_t>(qrow),
                                  &bars->q_full, pol_q);
        }
        last_q = static_cast<int>(nitem);
        for (int j = 0; j < it.nblk; ++j, ++gblk) {
          const int st = gblk % NST;
          const uint32_t use = gblk / NST;
          const bool gathered = j < it.nblk_g;
          const int64_t row = kv_row0 + (gathered ? static_cast<int64_t>(j) * BN
                                                  : it.win_lo + static_cast<int64_t>(j - it.nblk_g) * BN);
          if (gblk >= static_cast<uint32_t>(NST) &&
              !mbar_wait(&bars->k_empty[st], (use - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          sep::mbar_arrive_expect_tx(&bars->k_full[st], C::KV_BYTES);
#pragma unroll
          for (int r = 0; r < D / 64; ++r) {
            if (gathered)
              sep::tma_load_2d_hint(smem + C::OFF_K + st * C::KV_BYTES + r * C::REG, &tm_kc, r * 64,
                                    static_cast<int32_t>(row), &bars->k_full[st], pol_g);
            else
              sep::tma_load_2d(smem + C::OFF_K + st * C::KV_BYTES + r * C::REG, &tm_k, r * 64,
                               static_cast<int32_t>(row), &bars->k_full[st]);
          }
          last_k[st] = static_cast<int>(gblk);
          if (gblk >= static_cast<uint32_t>(NST) &&
              !mbar_wait(&bars->v_empty[st], (use - 1) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          sep::mbar_arrive_expect_tx(&bars->v_full[st], C::KV_BYTES);
#pragma unroll
          for (int r = 0; r < D / 64; ++r) {
            if (gathered)
              sep::tma_load_2d_hint(smem + C::OFF_V + st * C::KV_BYTES + r * C::REG, &tm_vc, r * 64,
                                    static_cast<int32_t>(row), &bars->v_full[st], pol_g);
            else
              sep::tma_load_2d(smem + C::OFF_V + st * C::KV_BYTES + r * C::REG, &tm_v, r * 64,
                               static_cast<int32_t>(row), &bars->v_full[st]);
          }
          last_v[st] = static_cast<int>(gblk);
        }
      }
      if (*abort) {
        // only the most recent load of each buffer can still be in flight
        if (last_q >= 0) drain_wait(&bars->q_full, last_q & 1);
        for (int s2 = 0; s2 < NST; ++s2) {
          if (last_k[s2] >= 0) drain_wait(&bars->k_full[s2], (last_k[s2] / NST) & 1);
          if (last_v[s2] >= 0) drain_wait(&bars->v_full[s2], (last_v[s2] / NST) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarpB) {
    // ------------------------------------------------------------ MMA issuers
    // Separate P (D = 64): one issuing thread per tile, so that a tile's S
    // and P*V wait only for that tile's softmax.  P over S (D = 128): one
    // thread issues both tiles, P*V of a tile before its next S.  The MMAs
    // of one thread complete in issue order; the barriers of the shared K,
    // V and Q stages take one commit from each issuer.
    if (!C::SEP_P) {
      if (warp == kMmaWarp && lane == 0) mma_single_issuer<D>(p, smem, tmem, bars, abort);
    } else if (lane == 0) {
      const int t = warp == kMmaWarp ? 0 : 1;
      constexpr uint32_t idesc_s = sep::idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_o = sep::idesc_bf16_f32(BM, D, true);
      // Shared-memory descriptors are built once: a K step only moves the
      // start address, whose field (bits 0-13, address >> 4) takes the
      // offset >> 4 without a carry (every address is below 256 KB).  Built
      // per instruction, the descriptor arithmetic of this single thread
      // costs about as much as the MMA itself.
      const uint64_t dq = sep::smem_desc_sw128(sep::smem_u32(smem + (t ? C::OFF_QB : C::OFF_QA)), 16);
      const uint64_t dk0 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_K), 16);
      const uint64_t dv0 = sep::smem_desc_sw128(sep::smem_u32(smem + C::OFF_V), C::REG);
      const uint32_t stm = tmem + (t ? C::COL_S1 : C::COL_S0);
      const uint32_t ptm = tmem + (t ? C::COL_P1 : C::COL_P0);
      const uint32_t otm = tmem + (t ? C::COL_O1 : C::COL_O0);
      uint32_t gblk = 0, nitem = 0, pphase = 0;
      uint32_t ns = 0;  // S products issued (separate-P protocol)
      bool ok = true;
      // O_t += P_t V (block `vblk` of the global stream); the first PV of an
      // item overwrites O_t, so it waits until the previous item's epilogue
      // of this tile has read O_t.
      auto issue_pv = [&](uint32_t vblk, bool first) -> bool {
        if (!mbar_wait(&bars->p_full[t], pphase, abort, p.err)) return false;
        pphase ^= 1u;
        if (!mbar_wait(&bars->v_full[vblk % NST], (vblk / NST) & 1, abort, p.err)) return false;
        if (first && nitem > 0 && !mbar_wait(&bars->o_empty[t], (nitem - 1) & 1, abort, p.err))
          return false;
        sep::tc_fence_after();
        const uint64_t dv = dv0 + static_cast<uint64_t>((vblk % NST) * (C::KV_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)  // 16 keys = 2048 bytes of V per step
          sep::mma_bf16_ts(otm, ptm + kk * 8, dv + kk * (2048 >> 4), idesc_o, (!first || kk > 0) ? 1u : 0u);
        if (C::SEP_P) sep::mma_commit(&bars->pv_done[t]);
        return true;
      };
      auto issue_s = [&](uint32_t kblk) -> bool {
        if (C::SEP_P) {
          // S_t is free once the softmax has read the previous block's scores
          if (ns > 0 && !mbar_wait(&bars->s_free[t], (ns - 1) & 1, abort, p.err)) return false;
          ++ns;
          sep::tc_fence_after();
        }
        const uint64_t dk = dk0 + static_cast<uint64_t>((kblk % NST) * (C::KV_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {  // 16 dims: 32 bytes within a 64-column region
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * C::REG + (kk % 4) * 32) >> 4);
          sep::mma_bf16_ss(stm, dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        sep::mma_commit(&bars->s_full[t]);
        return true;
      };
      for (; ok; ++nitem) {
        const int item = take_item<NST>(bars, nitem, p, abort, false);
        if (item < 0 || item >= p.n_items) break;
        const Item it = make_item(p, item);
        if (!mbar_wait(&bars->q_full, nitem & 1, abort, p.err)) break;
        bool prev = false;  // this tile kept the previous block
        bool pv = false;    // this tile already accumulated into O this item
        for (int j = 0; j < it.nblk; ++j, ++gblk) {
          if (!mbar_wait(&bars->k_full[gblk % NST], (gblk / NST) & 1, abort, p.err)) {
            ok = false;
            break;
          }
          sep::tc_fence_after();
          const bool act = block_active(it, t, j, p.S);
          if constexpr (C::SEP_P) {
            // S of block j (as soon as the softmax has read the previous
            // scores), then P*V of block j - 1 once its P is there
            if (act && !(ok = issue_s(gblk))) break;
            sep::mma_commit(&bars->k_empty[gblk % NST]);
            if (j == it.nblk - 1) sep::mma_commit(&bars->q_empty);
            if (prev) {
              if (!(ok = issue_pv(gblk - 1, !pv))) break;
              pv = true;
            }
            if (j > 0) sep::mma_commit(&bars->v_empty[(gblk - 1) % NST]);
          } else {
            // P is written over S: the previous block's P*V before this S
            if (prev) {
              if (!(ok = issue_pv(gblk - 1, !pv))) break;
              pv = true;
            }
            if (j > 0) sep::mma_commit(&bars->v_empty[(gblk - 1) % NST]);
            if (act) issue_s(gblk);
            sep::mma_commit(&bars->k_empty[gblk % NST]);
            if (j == it.nblk - 1) sep::mma_commit(&bars->q_empty);
          }
          prev = act;
        }
        if (!ok) break;
        // last block's P*V, then hand O to the epilogue
        if (prev && !(ok = issue_pv(gblk - 1, !pv))) break;
        sep::mma_commit(&bars->o_full[t]);
        sep::mma_commit(&bars->v_empty[(gblk - 1) % NST]);
      }
      sep::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax (tile t)
    const int t = warp >> 2;            // 0: tile A, 1: tile B
    const int row = threadIdx.x & 127;  // tile row == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t s_col = tmem + lane_base + (t ? C::COL_S1 : C::COL_S0);
    const uint32_t p_col = tmem + lane_base + (t ? C::COL_P1 : C::COL_P0);
    const uint32_t o_col = tmem + lane_base + (t ? C::COL_O1 : C::COL_O0);
    uint32_t sphase = 0, nitem = 0;
    uint32_t npv = 0;  // P*V products of this tile issued so far (separate-P protocol)
    // Separate-P protocol, after the scores of a block are in registers:
    // free S_t for the next block's MMA, then wait until the previous P*V
    // (reader of P_t, writer of O_t) is done.
    auto s_read_pv_wait = [&]() -> bool {
      if constexpr (C::SEP_P) {
        sep::tc_fence_before();
        sep::mbar_arrive(&bars->s_free[t]);
        if (npv > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[t], (npv - 1) & 1, abort, p.err)))
          return false;
        ++npv;
        sep::tc_fence_after();
      }
      return true;
    };
    bool ok = true;
    for (; ok; ++nitem) {
      const int item = take_item<NST>(bars, nitem, p, abort, true);
      if (item < 0 || item >= p.n_items) break;
      const Item it = make_item(p, item);
      // this tile's scalars (the rest of the item is not needed here)
      const int my_q0 = t ? it.q0[1] : it.q0[0];
      const int my_lo = t ? it.lo[1] : it.lo[0];
      const int my_nG = t ? it.nG[1] : it.nG[0];
      const int my_last = my_q0 + BM - 1 < p.S - 1 ? my_q0 + BM - 1 : p.S - 1;
      const int nblk_g = it.nblk_g, nblk = it.nblk, win_lo = it.win_lo;
      const int h = t ? it.h[1] : it.h[0];
      const int b = it.b;
      const int i = my_q0 + row;
      const int ie = i < p.S ? i : p.S - 1;  // rows past the end mask like the last row
      const uint8_t* flags = p.is_sep + static_cast<int64_t>(b) * p.S;
      float m_ref = -INFINITY, l = 0.f;
      // separator-or-initial flags of 4 positions (base + 32c + lane) per lane,
      // loaded one window block ahead of their use
      auto load_flags = [&](int base) -> uint32_t {
        uint32_t f = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int pos = base + 32 * c + lane;
          if (pos < p.S && (flags[pos] != 0 || pos < p.a)) f |= 1u << c;
        }
        return f;
      };
      uint32_t fl_next = load_flags(win_lo), fl_cur = 0;
      for (int j = 0; j < nblk; ++j) {
        if (j >= nblk_g) {
          fl_cur = fl_next;
          if (j + 1 < nblk) fl_next = load_flags(win_lo + (j + 1 - nblk_g) * BN);
        }
        // skip blocks this tile keeps nothing of (see block_active)
        if (j < nblk_g ? j * BN >= my_nG
                       : (win_lo + (j - nblk_g) * BN > my_last ||
                          win_lo + (j - nblk_g) * BN + BN - 1 < my_lo))
          continue;
        uint32_t keep[4];
        if (j < nblk_g) {
          const int valid = my_nG - j * BN;
#pragma unroll
          for (int c = 0; c < 4; ++c) keep[c] = bits_le(valid - 1 - 32 * c);
        } else {
          const int base = win_lo + (j - nblk_g) * BN;
          const int ihi = ie - base, ilo = ie - p.n - base, jlo = my_lo - base;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint32_t sepbits = __ballot_sync(0xffffffffu, (fl_cur >> c) & 1u);
            keep[c] = bits_le(ihi - 32 * c) & (~bits_le(ilo - 32 * c) | sepbits) &
                      ~bits_le(jlo - 1 - 32 * c);
          }
        }
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[t], sphase, abort, p.err))) {
          ok = false;
          break;
        }
        sphase ^= 1;
        sep::tc_fence_after();
        // Fast path (after the block where a row first saw a key): one pass
        // over S against the reference m_ref, P kept in registers until the
        // block's row sum is known to stay within 2^16.  Otherwise (first
        // block, or scores that grew too far): the exact two-pass path, which
        // moves the reference to the block maximum when that exceeds it by
        // more than 2^8 and rescales O.
        bool fast_done = false;
        uint32_t ra[32], rb[32];
        sep::tmem_ld32(s_col, ra);
        sep::tmem_wait_ld_r32(ra);
        // A row without a reference yet (its first kept block) takes the
        // maximum of its kept scores among the first 32 keys: never above the
        // block maximum, so P cannot underflow, and the row-sum test below
        // catches a reference that is too low.
        float m_use = m_ref;
        if (__any_sync(0xffffffffu, m_ref == -INFINITY)) {
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mx[e & 3] = fmaxf(mx[e & 3], (keep[0] >> e) & 1u ? __uint_as_float(ra[e]) : -INFINITY);
          const float m0 = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
          if (m_ref == -INFINITY) m_use = m0 * p.scale_log2;
        }
        if (__all_sync(0xffffffffu, m_use != -INFINITY)) {
          uint32_t pk[64];
          float2 sm2[4];  // partial row sums, four independent pairs
#pragma unroll
          for (int u = 0; u < 4; ++u) sm2[u] = make_float2(0.f, 0.f);
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 nm2 = make_float2(-m_use, -m_use);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t* cur = (c & 1) ? rb : ra;
            uint32_t* nxt = (c & 1) ? ra : rb;
            if (c < 3) sep::tmem_ld32(s_col + 32 * (c + 1), nxt);  // overlaps this group's math
            const uint32_t kc = keep[c];
            if (__all_sync(0xffffffffu, kc == 0u)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) pk[16 * c + e] = 0u;
            } else if (__all_sync(0xffffffffu, kc == 0xffffffffu)) {
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float2 y = sep::ffma2(make_float2(__uint_as_float(cur[e]), __uint_as_float(cur[e + 1])), sc2, nm2);
                const float2 pp = make_float2(sep::ex2_approx(y.x), sep::ex2_approx(y.y));
                sm2[(e >> 1) & 3] = sep::fadd2(sm2[(e >> 1) & 3], pp);
                pk[16 * c + (e >> 1)] = sep::pack_bf16x2(pp.x, pp.y);
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                const float x0 = (kc >> e) & 1u ? __uint_as_float(cur[e]) : -INFINITY;
                const float x1 = (kc >> (e + 1)) & 1u ? __uint_as_float(cur[e + 1]) : -INFINITY;
                const float2 y = sep::ffma2(make_float2(x0, x1), sc2, nm2);
                const float2 pp = make_float2(sep::ex2_approx(y.x), sep::ex2_approx(y.y));
                sm2[(e >> 1) & 3] = sep::fadd2(sm2[(e >> 1) & 3], pp);
                pk[16 * c + (e >> 1)] = sep::pack_bf16x2(pp.x, pp.y);
              }
            }
            if (c < 3) sep::tmem_wait_ld_r32(nxt);
          }
          const float2 s01 = sep::fadd2(sm2[0], sm2[1]), s23 = sep::fadd2(sm2[2], sm2[3]);
          const float rowsum = (s01.x + s01.y) + (s23.x + s23.y);
          // Every P of the block is at most its row sum: up to 2^16 (P in
          // bf16, O and l in fp32) the block stays on the reference m_ref; an
          // overflow or a NaN fails the test as well, and the exact path
          // below moves the reference instead.
          if (!__any_sync(0xffffffffu, !(rowsum <= 65536.f))) {
            m_ref = m_use;
            l += rowsum;
            if (!s_read_pv_wait()) {
              ok = false;
              break;
            }
            sep::tmem_st32(p_col, pk);
            sep::tmem_st32(p_col + 32, pk + 32);
            fast_done = true;
          }
        }
        if (!fast_done) {
          // pass 1: masked row maximum of the raw scores (8 independent chains)
          float mx[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) mx[u] = -INFINITY;
          // (loops over the 4 column groups stay rolled: one group of scores in
          // registers at a time; the keep words rotate instead of being indexed)
          uint32_t k0 = keep[0], k1 = keep[1], k2 = keep[2], k3 = keep[3];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            if (__any_sync(0xffffffffu, k0 != 0u)) {
              uint32_t r[32];
              sep::tmem_ld32(s_col + 32 * c, r);
              sep::tmem_wait_ld_r32(r);
#pragma unroll
              for (int e = 0; e < 32; ++e)
                mx[e & 7] = fmaxf(mx[e & 7], (k0 >> e) & 1u ? __uint_as_float(r[e]) : -INFINITY);
            }
            k0 = k1;
            k1 = k2;
            k2 = k3;
          }
          const float mblk = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                             p.scale_log2;
          float alpha = 1.f;
          const bool grow = mblk > m_ref + kRescaleLog2;
          if (grow) {
            alpha = sep::ex2_approx(m_ref - mblk);  // 0 while m_ref is -inf
            m_ref = mblk;
          }
          // D = 128: S_t of this block was issued after this tile's previous
          // P*V, and MMAs complete in order, so that P*V is done.  Separate P:
          // wait for it (pass 2 below still reads S_t; it is freed after).
          if constexpr (C::SEP_P) {
            if (npv > 0 && !__all_sync(0xffffffffu, mbar_wait(&bars->pv_done[t], (npv - 1) & 1, abort, p.err))) {
              ok = false;
              break;
            }
            sep::tc_fence_after();
          }
          if (j > 0 && __any_sync(0xffffffffu, grow)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              sep::tmem_ld32(o_col + 32 * c, o);
              sep::tmem_wait_ld_r32(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              sep::tmem_st32(o_col + 32 * c, o);
            }
          }
          const float mr = m_ref == -INFINITY ? 0.f : m_ref;
          float sm[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) sm[u] = 0.f;
          // pass 2: P = 2^(s*scale - m) as bf16 pairs written over S_t: keys
          // [32c, 32c+32) go to columns [16c, 16c+16), which hold scores of
          // keys already read back
          k0 = keep[0];
          k1 = keep[1];
          k2 = keep[2];
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            if (!__any_sync(0xffffffffu, k0 != 0u)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) r[e] = 0u;
              sep::tmem_st16(p_col + 16 * c, r);
              k0 = k1;
              k1 = k2;
              k2 = keep[3];
              continue;
            }
            sep::tmem_ld32(s_col + 32 * c, r);
            sep::tmem_wait_ld_r32(r);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const float x0 = (k0 >> e) & 1u ? __uint_as_float(r[e]) : -INFINITY;
              const float x1 = (k0 >> (e + 1)) & 1u ? __uint_as_float(r[e + 1]) : -INFINITY;
              const float p0 = sep::ex2_approx(fmaf(x0, p.scale_log2, -mr));
              const float p1 = sep::ex2_approx(fmaf(x1, p.scale_log2, -mr));
              sm[e & 7] += p0;
              sm[(e + 1) & 7] += p1;
              r[e >> 1] = sep::pack_bf16x2(p0, p1);
            }
            sep::tmem_st16(p_col + 16 * c, r);
            k0 = k1;
            k1 = k2;
            k2 = keep[3];
          }
          l = l * alpha + (((sm[0] + sm[1]) + (sm[2] + sm[3])) + ((sm[4] + sm[5]) + (sm[6] + sm[7])));
          if constexpr (C::SEP_P) {
            // every score of the block has been read: free S_t (the previous
            // P*V was waited for above)
            sep::tmem_wait_st();
            sep::tc_fence_before();
            sep::mbar_arrive(&bars->s_free[t]);
            ++npv;
          }
        }
        sep::tmem_wait_st();
        sep::tc_fence_before();
        sep::mbar_arrive(&bars->p_full[t]);
      }
      if (!ok) break;
      // epilogue: O_t / l -> out (bf16), lse
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_full[t], nitem & 1, abort, p.err))) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      const float inv = 1.f / l;
      if (C::STG_BYTES > 0 && my_q0 + BM <= p.S) {
        // whole tile: rows into a 128-byte swizzled staging tile (16-byte
        // unit u of row r at u ^ (r & 7): one row per thread, conflict-free),
        // then one tensor store.  A thread per row writing global memory
        // directly touches 32 lines per warp instruction.
        uint8_t* stg = smem + C::OFF_STG + t * C::Q_BYTES;
        if (row == 0) sep::bulk_wait_read0();  // the previous store has read the tile
        sep::named_bar_sync(1 + t, 128);
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          sep::tmem_ld32(o_col + 32 * c, o);
          sep::tmem_wait_ld_r32(o);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = sep::pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            w.y = sep::pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            w.z = sep::pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            w.w = sep::pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            const int u = 4 * c + q;
            *reinterpret_cast<uint4*>(stg + row * 128 + ((u ^ (row & 7)) << 4)) = w;
          }
        }
        sep::fence_proxy_async_smem();
        sep::named_bar_sync(1 + t, 128);
        if (row == 0) {
          sep::tma_store_2d_hint(&tm_o, 0, static_cast<int32_t>(static_cast<int64_t>(b * p.Hq + h) * p.S + my_q0),
                                 stg, sep::l2_evict_first_policy());
          sep::bulk_commit();
        }
      } else {
      __nv_bfloat16* orow = p.out + (static_cast<int64_t>(b * p.Hq + h) * p.S + i) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        sep::tmem_ld32(o_col + 32 * c, o);
        sep::tmem_wait_ld_r32(o);
        if (i < p.S) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = sep::pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            w.y = sep::pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            w.z = sep::pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            w.w = sep::pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            __stcs(reinterpret_cast<uint4*>(orow + 32 * c + 8 * q), w);  // streamed out
          }
        }
      }
      }
      if (p.lse && i < p.S)
        __stcs(p.lse + static_cast<int64_t>(b * p.Hq + h) * p.S + i, (m_ref + __log2f(l)) * 0.69314718055994530942f);
      sep::tc_fence_before();
      sep::mbar_arrive(&bars->o_empty[t]);
    }
    if (C::STG_BYTES > 0 && row == 0) sep::bulk_wait0();  // output stores done before exit
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  if (warp == kMmaWarp) {
    __syncwarp();
    sep::tmem_dealloc(tmem, kTmemCols);
  }
}

// Copy, per (b, kv head), the K/V rows of the initial tokens [0, min(a, S))
// followed by every separator at a position >= a into the compact buffers
// Kc/Vc [B, Hkv, S, D]; rows from the end of that list up to 128 (at least)
// and up to the next multiple of 128 are zero-filled, so whole 128-row tiles
// read finite values.  One CTA copies 64 rows.  The first thread also zeroes
// the attention kernel's work-item counter (every earlier kernel on the
// stream, the previous attention launch included, has completed here).
template <int D>
__global__ void __launch_bounds__(256) k_gather_sep_rows(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ prefix, const int32_t* __restrict__ idx, int Hkv, int S, int a,
    __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc, int32_t* err,
    int32_t* __restrict__ sched) {
  constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the index's producer
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0) *sched = 0;
  const int g = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * 64;
  const int32_t* pre = prefix + static_cast<int64_t>(b) * (S + 1);
  const int aa = a < S ? a : S;
  const int sep_begin = pre[aa];
  const int total = aa + (pre[S] - sep_begin);
  int lim = ((total + BN - 1) / BN) * BN;
  if (lim < BN) lim = BN;
  if (lim > S) lim = S;
  if (r0 >= lim) return;
  const int64_t base = static_cast<int64_t>(b * Hkv + g) * S;
  const int32_t* ix = idx + static_cast<int64_t>(b) * S;
  for (int e = threadIdx.x; e < 64 * CH; e += 256) {
    const int r = r0 + e / CH, c = e % CH;
    if (r >= lim) break;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (r < total) {
      const int pos = r < aa ? r : ix[sep_begin + (r - aa)];
      if (pos >= 0 && pos < S) {
        kv = reinterpret_cast<const uint4*>(k + (base + pos) * D)[c];
        vv = reinterpret_cast<const uint4*>(v + (base + pos) * D)[c];
      } else if (err) {
        atomicOr(err, sep::ERR_BAD_INDEX);
      }
    }
    reinterpret_cast<uint4*>(kc + (base + r) * D)[c] = kv;
    reinterpret_cast<uint4*>(vc + (base + r) * D)[c] = vv;
  }
}

// ------------------------------------------------------------------ host

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_map(CUtensorMap* m, const void* base, int64_t rows, int D) {
  return sep::make_rows_map(m, base, rows, D, 128);
}

int num_sms() {
  static int sms[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (!sms[dev]) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    sms[dev] = v > 0 ? v : 148;
  }
  return sms[dev];
}

template <int D>
int launch(const void* q, const void* k, const void* v, const uint8_t* is_sep,
           const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int a, int n,
           float scale, void* out, float* lse, void* kc, void* vc, int32_t* sched, cudaStream_t st) {
  using C = Cfg<D>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(k_prefill_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::ALLOC) != cudaSuccess)
      return SEP_ECUDA;
    attr_set[dev] = true;
  }
  const int64_t qrows = static_cast<int64_t>(B) * Hq * S;
  const int64_t krows = static_cast<int64_t>(B) * Hkv * S;
  if (qrows >= (1ll << 31) || krows >= (1ll << 31)) return SEP_EINVAL;
  CUtensorMap mq, mk, mv, mkc, mvc, mo;
  if (!make_map(&mq, q, qrows, D) || !make_map(&mo, out, qrows, D) || !make_map(&mk, k, krows, D) ||
      !make_map(&mv, v, krows, D) ||
      !make_map(&mkc, kc, krows, D) || !make_map(&mvc, vc, krows, D))
    return SEP_ECUDA;

  dim3 ggrid((S + 63) / 64, Hkv, B);
  if (sep::launch_pdl(k_gather_sep_rows<D>, ggrid, dim3(256), 0, st,
                      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                      prefix, idx, Hkv, S, a, static_cast<__nv_bfloat16*>(kc),
                      static_cast<__nv_bfloat16*>(vc), sep::device_error_word(), sched) != cudaSuccess)
    return SEP_ECUDA;

  Params p;
  p.is_sep = is_sep;
  p.prefix = prefix;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.a = a;
  p.n = n;
  p.G = Hq / Hkv;
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  if (p.pair_heads) {
    p.npairs = Hq / 2;
    p.ntiles_item = (S + BM - 1) / BM;
  } else {
    p.npairs = Hq;
    p.ntiles_item = (S + 2 * BM - 1) / (2 * BM);
  }
  const int64_t items = static_cast<int64_t>(p.ntiles_item) * B * p.npairs;
  if (items >= (1ll << 31)) return SEP_EINVAL;
  p.n_items = static_cast<int>(items);
  p.scale_log2 = scale * 1.44269504088896340736f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = sep::device_error_word();
  p.sched = sched;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  if (sep::launch_pdl(k_prefill_tc<D>, dim3(grid), dim3(kThreads), C::ALLOC, st, mq, mk, mv, mkc,
                      mvc, mo, p) != cudaSuccess)
    return SEP_ECUDA;
  return sep::launch_status();
}

}  // namespace

namespace sep {
// Workspace: 256 bytes of head (the work-item counter) and the compact K and
// V row lists.
size_t prefill_tc_workspace(int B, int Hkv, int S, int D) {
  return 256 + 2 * ((static_cast<size_t>(B) * Hkv * S * D * 2 + 255) / 256 * 256);
}

int prefill_tc(const void* q, const void* k, const void* v, const uint8_t* is_sep,
               const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int D,
               int a, int n, float scale, void* out, float* lse, void* workspace, cudaStream_t st) {
  const size_t half = (static_cast<size_t>(B) * Hkv * S * D * 2 + 255) / 256 * 256;
  int32_t* sched = static_cast<int32_t*>(workspace);
  void* kc = static_cast<uint8_t*>(workspace) + 256;
  void* vc = static_cast<uint8_t*>(kc) + half;
  if (D == 64)
    return launch<64>(q, k, v, is_sep, prefix, idx, B, Hq, Hkv, S, a, n, scale, out, lse, kc, vc,
                      sched, st);
  if (D == 128)
    return launch<128>(q, k, v, is_sep, prefix, idx, B, Hq, Hkv, S, a, n, scale, out, lse, kc, vc,
                       sched, st);
  return SEP_EDTYPE;
}
}  // namespace sep

namespace sep {
bool make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows < 1 || box_rows < 1 || box_rows > 256) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace sep
