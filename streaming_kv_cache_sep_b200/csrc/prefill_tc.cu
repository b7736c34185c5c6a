// bf16 Sep-Attention prefill on tcgen05 tensor cores (sm_100a).
//
// What it computes ("HKUDS047: SepLLM ..." study, section "SepAttention";
// jieyibu.net explainer, section 1.2): for query row i,
//   out_i = sum_{j in K_i} softmax(scale * q_i . k_j) v_j,
//   K_i = { j <= i : j < a  or  is_sep[j]  or  i - j < n }.
//
// How.  A CTA owns one (batch b, query head h, tile of 128 query rows
// [q0, q0+128)).  With lo = max(0, q0 - n + 1) every kept key of every row
// of the tile lies in one of two sets:
//   * the gathered set: initial tokens [0, min(a, lo)) and the separators in
//     [a, lo).  These are kept by every row of the tile, so their blocks need
//     no element mask.  A small kernel first copies, per (b, kv head), the
//     K/V rows of the initial tokens followed by all separators at positions
//     >= a into a contiguous workspace buffer; the gathered set of any tile is
//     then a prefix of that buffer, and is loaded with plain TMA tiles.
//   * the window range [lo, q0 + 128), loaded contiguously from K/V.  Its
//     blocks carry the element mask  j <= i and (i - j < n or is_sep[j] or
//     j < a), which handles separators that sit inside some rows' windows.
// Each key of K_i is therefore scored exactly once.
//
// Warp roles (192 threads): warps 0-3 run the softmax, one thread per query
// row (TMEM lane = row); warp 4 issues TMA loads; warp 5 owns TMEM and issues
// the tcgen05.mma instructions.  S = Q K^T goes to one of two 128-column TMEM
// buffers, so the MMA for block j+1 overlaps the softmax of block j.  P is
// rounded to bf16 into a 128-byte-swizzled shared tile and O += P V
// accumulates in TMEM.  The running maximum is only moved (and O rescaled)
// when it grows by more than 2^8, so P stays <= 256.
#include <string.h>

#include "common.cuh"

namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // keys per block
constexpr int NST = 2;   // K/V shared-memory stages
constexpr int kThreads = 192;
constexpr int kTmaWarp = 4;
constexpr int kMmaWarp = 5;
constexpr uint32_t kTmemCols = 512;  // S0 | S1 | O
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct Layout {
  static constexpr int REG = 128 * 128;        // one 64-column region of a 128-row tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;  // one K (or V) stage
  static constexpr int P_BYTES = BM * BN * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + NST * KV_BYTES;
  static constexpr int OFF_P = OFF_V + NST * KV_BYTES;
  static constexpr int OFF_BAR = OFF_P + P_BYTES;
  static constexpr int BYTES = OFF_BAR + 256;
  // +1024 slack for 1024-byte alignment; at least 120 KB so that one CTA
  // (which owns all 512 TMEM columns) runs per SM
  static constexpr int ALLOC = BYTES + 1024 > 120 * 1024 ? BYTES + 1024 : 120 * 1024;
};

struct Bars {
  uint64_t k_full[NST], k_empty[NST], v_full[NST], v_empty[NST];
  uint64_t s_full[2], p_full, o_done, drain;
  uint32_t tmem_base;
  int abort;
};

struct Params {
  const uint8_t* is_sep;
  const int32_t* prefix;
  int B, Hq, Hkv, S, a, n, G, ntiles;
  float scale_log2;
  __nv_bfloat16* out;
  float* lse;
  int32_t* err;
};

// mask of bit positions c in [0, 32) with c <= x
__device__ __forceinline__ uint32_t bits_le(int x) {
  return x < 0 ? 0u : (x >= 31 ? 0xffffffffu : (0xffffffffu >> (31 - x)));
}

// Wait without the abort short-cut (used only to drain in-flight copies or
// MMAs before the CTA exits after an abort).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  int dummy = 0;
  sep::mbar_wait(bar, parity, &dummy, nullptr);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    k_prefill_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kc,
                 const __grid_constant__ CUtensorMap tm_vc, const Params p) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + L::OFF_BAR);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = p.ntiles - 1 - static_cast<int>(blockIdx.x);  // heaviest tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int g = h / p.G;
  const int S = p.S;
  const int q0 = qt * BM;
  const int q1 = q0 + BM < S ? q0 + BM : S;
  const int lo = q0 - p.n + 1 > 0 ? q0 - p.n + 1 : 0;
  const int32_t* pre = p.prefix + static_cast<int64_t>(b) * (S + 1);
  const int aa = p.a < S ? p.a : S;
  const int n_init = p.a < lo ? p.a : lo;
  const int n_sep = lo > aa ? pre[lo] - pre[aa] : 0;
  const int nG = n_init + n_sep;                 // gathered keys (prefix of the compact buffer)
  const int nblk_g = (nG + BN - 1) / BN;
  const int nblk_w = (q1 - lo + BN - 1) / BN;
  const int nblk = nblk_g + nblk_w;
  const int64_t kv_row0 = static_cast<int64_t>(b * p.Hkv + g) * S;  // row of key 0 in K/V/Kc/Vc

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      sep::mbar_init(&bars->k_full[s], 1);
      sep::mbar_init(&bars->k_empty[s], 1);
      sep::mbar_init(&bars->v_full[s], 1);
      sep::mbar_init(&bars->v_empty[s], 1);
    }
    sep::mbar_init(&bars->s_full[0], 1);
    sep::mbar_init(&bars->s_full[1], 1);
    sep::mbar_init(&bars->p_full, 128);
    sep::mbar_init(&bars->o_done, 1);
    sep::mbar_init(&bars->drain, 1);
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

  if (warp == kTmaWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      sep::tma_prefetch_desc(&tm_q);
      sep::tma_prefetch_desc(&tm_k);
      sep::tma_prefetch_desc(&tm_v);
      sep::tma_prefetch_desc(&tm_kc);
      sep::tma_prefetch_desc(&tm_vc);
      int last_k[NST], last_v[NST];  // last block loaded into each stage
      for (int s2 = 0; s2 < NST; ++s2) last_k[s2] = last_v[s2] = -1;
      for (int j = 0; j < nblk; ++j) {
        const int st = j % NST;
        const uint32_t use = j / NST;
        const bool gathered = j < nblk_g;
        const CUtensorMap* mk = gathered ? &tm_kc : &tm_k;
        const CUtensorMap* mv = gathered ? &tm_vc : &tm_v;
        const int64_t row = kv_row0 + (gathered ? static_cast<int64_t>(j) * BN
                                                : lo + static_cast<int64_t>(j - nblk_g) * BN);
        if (j >= NST && !sep::mbar_wait(&bars->k_empty[st], (use - 1) & 1, abort, p.err)) break;
        uint8_t* sk = smem + L::OFF_K + st * L::KV_BYTES;
        if (j == 0) {
          sep::mbar_arrive_expect_tx(&bars->k_full[0], L::KV_BYTES + L::Q_BYTES);
          const int64_t qrow = static_cast<int64_t>(b * p.Hq + h) * S + q0;
#pragma unroll
          for (int r = 0; r < D / 64; ++r)
            sep::tma_load_2d(smem + L::OFF_Q + r * L::REG, &tm_q, r * 64, static_cast<int32_t>(qrow),
                             &bars->k_full[0]);
        } else {
          sep::mbar_arrive_expect_tx(&bars->k_full[st], L::KV_BYTES);
        }
#pragma unroll
        for (int r = 0; r < D / 64; ++r)
          sep::tma_load_2d(sk + r * L::REG, mk, r * 64, static_cast<int32_t>(row), &bars->k_full[st]);
        last_k[st] = j;
        if (j >= NST && !sep::mbar_wait(&bars->v_empty[st], (use - 1) & 1, abort, p.err)) break;
        uint8_t* sv = smem + L::OFF_V + st * L::KV_BYTES;
        sep::mbar_arrive_expect_tx(&bars->v_full[st], L::KV_BYTES);
#pragma unroll
        for (int r = 0; r < D / 64; ++r)
          sep::tma_load_2d(sv + r * L::REG, mv, r * 64, static_cast<int32_t>(row), &bars->v_full[st]);
        last_v[st] = j;
      }
      if (*abort) {
        // Only the last load of each stage can still be in flight (a stage is
        // reloaded only after its previous contents were consumed): let those
        // land before the CTA's shared memory goes away.
        for (int s2 = 0; s2 < NST; ++s2) {
          if (last_k[s2] >= 0) drain_wait(&bars->k_full[s2], (last_k[s2] / NST) & 1);
          if (last_v[s2] >= 0) drain_wait(&bars->v_full[s2], (last_v[s2] / NST) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = sep::idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idesc_o = sep::idesc_bf16_f32(BM, D, true);
      const uint32_t sq = sep::smem_u32(smem + L::OFF_Q);
      const uint32_t sp = sep::smem_u32(smem + L::OFF_P);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj % NST;
        if (!sep::mbar_wait(&bars->p_full, jj & 1, abort, p.err)) return false;
        if (!sep::mbar_wait(&bars->v_full[st], (jj / NST) & 1, abort, p.err)) return false;
        sep::tc_fence_after();
        const uint32_t sv = sep::smem_u32(smem + L::OFF_V + st * L::KV_BYTES);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t ad = sep::smem_desc_sw128(sp + (kk / 4) * L::REG + (kk % 4) * 32, 16);
          const uint64_t bd = sep::smem_desc_sw128(sv + kk * 2048, L::REG);
          sep::mma_bf16_ss(tmem + 256, ad, bd, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        sep::mma_commit(&bars->o_done);
        sep::mma_commit(&bars->v_empty[st]);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j % NST;
        if (!sep::mbar_wait(&bars->k_full[st], (j / NST) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        sep::tc_fence_after();
        const uint32_t sk = sep::smem_u32(smem + L::OFF_K + st * L::KV_BYTES);
        const uint32_t s_tmem = tmem + (j & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sep::smem_desc_sw128(sq + (kk / 4) * L::REG + (kk % 4) * 32, 16);
          const uint64_t bd = sep::smem_desc_sw128(sk + (kk / 4) * L::REG + (kk % 4) * 32, 16);
          sep::mma_bf16_ss(s_tmem, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        sep::mma_commit(&bars->s_full[j & 1]);
        sep::mma_commit(&bars->k_empty[st]);
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(nblk - 1);
      // every MMA issued above has completed once `drain` fires
      sep::mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int t = threadIdx.x;  // tile row == TMEM lane
    const int i = q0 + t;
    const int ie = i < S ? i : S - 1;  // rows past the end mask like the last row
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint8_t* flags = p.is_sep + static_cast<int64_t>(b) * S;
    float m_ref = -INFINITY, l = 0.f;
    uint8_t* sp_row = smem + L::OFF_P + (t >> 3) * 1024 + (t & 7) * 128;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      // keep-bits of this row for the block's 128 columns
      uint32_t keep[4];
      if (j < nblk_g) {
        const int valid = nG - j * BN;
#pragma unroll
        for (int c = 0; c < 4; ++c) keep[c] = bits_le(valid - 1 - 32 * c);
      } else {
        const int base = lo + (j - nblk_g) * BN;
        const int ihi = ie - base, ilo = ie - p.n - base;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int pos = base + 32 * c + lane;
          const bool f = pos < S && (flags[pos] != 0 || pos < p.a);
          const uint32_t sepbits = __ballot_sync(0xffffffffu, f);
          keep[c] = bits_le(ihi - 32 * c) & (~bits_le(ilo - 32 * c) | sepbits);
        }
      }
      if (!__all_sync(0xffffffffu, sep::mbar_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort, p.err))) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      uint32_t r[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) sep::tmem_ld32(tmem + lane_base + (j & 1) * 128 + 32 * c, r[c]);
      sep::tmem_wait_ld();
      float mblk = -INFINITY;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x = (keep[c] >> e) & 1u ? __uint_as_float(r[c][e]) * p.scale_log2 : -INFINITY;
          r[c][e] = __float_as_uint(x);
          mblk = fmaxf(mblk, x);
        }
      float alpha = 1.f;
      const bool grow = mblk > m_ref + kRescaleLog2;
      if (grow) {
        alpha = sep::ex2_approx(m_ref - mblk);  // 0 while m_ref is -inf
        m_ref = mblk;
      }
      const float mr = m_ref == -INFINITY ? 0.f : m_ref;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c)
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float pe = sep::ex2_approx(__uint_as_float(r[c][e]) - mr);
          r[c][e] = __float_as_uint(pe);
          sum += pe;
        }
      l = l * alpha + sum;
      // the previous P*V must be done before P is overwritten or O rescaled
      if (j >= 1) {
        if (!__all_sync(0xffffffffu, sep::mbar_wait(&bars->o_done, (j - 1) & 1, abort, p.err))) {
          ok = false;
          break;
        }
        sep::tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            const uint32_t ta = tmem + lane_base + 256 + 32 * c;
            sep::tmem_ld32(ta, o);
            sep::tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            sep::tmem_st32(ta, o);
          }
          sep::tmem_wait_st();
        }
      }
      // P row -> shared memory, bf16, 128-byte swizzle (two 64-key regions)
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int c = ch >> 2, e0 = (ch & 3) * 8;
        uint4 w;
        w.x = sep::pack_bf16x2(__uint_as_float(r[c][e0 + 0]), __uint_as_float(r[c][e0 + 1]));
        w.y = sep::pack_bf16x2(__uint_as_float(r[c][e0 + 2]), __uint_as_float(r[c][e0 + 3]));
        w.z = sep::pack_bf16x2(__uint_as_float(r[c][e0 + 4]), __uint_as_float(r[c][e0 + 5]));
        w.w = sep::pack_bf16x2(__uint_as_float(r[c][e0 + 6]), __uint_as_float(r[c][e0 + 7]));
        const int region = ch >> 3, cc = ch & 7;
        *reinterpret_cast<uint4*>(sp_row + region * L::REG + ((cc ^ (t & 7)) << 4)) = w;
      }
      sep::fence_proxy_async_smem();
      sep::tc_fence_before();
      sep::mbar_arrive(&bars->p_full);
    }
    // epilogue: O / l -> out (bf16), lse
    if (ok && __all_sync(0xffffffffu, sep::mbar_wait(&bars->o_done, (nblk - 1) & 1, abort, p.err))) {
      sep::tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = p.out + (static_cast<int64_t>(b * p.Hq + h) * S + i) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        sep::tmem_ld32(tmem + lane_base + 256 + 32 * c, o);
        sep::tmem_wait_ld();
        if (i < S) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = sep::pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
            w.y = sep::pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
            w.z = sep::pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
            w.w = sep::pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * c + 8 * q) = w;
          }
        }
      }
      if (p.lse && i < S)
        p.lse[static_cast<int64_t>(b * p.Hq + h) * S + i] =
            (m_ref + __log2f(l)) * 0.69314718055994530942f;
    }
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
// read finite values.  One CTA copies 64 rows.
template <int D>
__global__ void __launch_bounds__(256) k_gather_sep_rows(
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ prefix, const int32_t* __restrict__ idx, int Hkv, int S, int a,
    __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc, int32_t* err) {
  constexpr int CH = D * 2 / 16;  // 16-byte chunks per row
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

// 2-D bf16 view [rows, D] with 128-byte swizzled boxes of 64 columns x 128 rows.
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int D) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D>
int launch(const void* q, const void* k, const void* v, const uint8_t* is_sep,
           const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int a, int n,
           float scale, void* out, float* lse, void* kc, void* vc, cudaStream_t st) {
  using L = Layout<D>;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(k_prefill_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             L::ALLOC) != cudaSuccess)
      return SEP_ECUDA;
    attr_set[dev] = true;
  }
  const int64_t qrows = static_cast<int64_t>(B) * Hq * S;
  const int64_t krows = static_cast<int64_t>(B) * Hkv * S;
  if (qrows >= (1ll << 31) || krows >= (1ll << 31)) return SEP_EINVAL;
  CUtensorMap mq, mk, mv, mkc, mvc;
  if (!make_map(&mq, q, qrows, D) || !make_map(&mk, k, krows, D) || !make_map(&mv, v, krows, D) ||
      !make_map(&mkc, kc, krows, D) || !make_map(&mvc, vc, krows, D))
    return SEP_ECUDA;

  dim3 ggrid((S + 63) / 64, Hkv, B);
  k_gather_sep_rows<D><<<ggrid, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v), prefix, idx, Hkv,
      S, a, static_cast<__nv_bfloat16*>(kc), static_cast<__nv_bfloat16*>(vc),
      sep::device_error_word());
  if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;

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
  p.ntiles = (S + BM - 1) / BM;
  p.scale_log2 = scale * 1.44269504088896340736f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.err = sep::device_error_word();
  dim3 grid(p.ntiles, Hq, B);
  k_prefill_tc<D><<<grid, kThreads, L::ALLOC, st>>>(mq, mk, mv, mkc, mvc, p);
  return sep::launch_status();
}

}  // namespace

namespace sep {
size_t prefill_tc_workspace(int B, int Hkv, int S, int D) {
  return 2 * ((static_cast<size_t>(B) * Hkv * S * D * 2 + 255) / 256 * 256);
}

int prefill_tc(const void* q, const void* k, const void* v, const uint8_t* is_sep,
               const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int D,
               int a, int n, float scale, void* out, float* lse, void* workspace, cudaStream_t st) {
  const size_t half = (static_cast<size_t>(B) * Hkv * S * D * 2 + 255) / 256 * 256;
  void* kc = workspace;
  void* vc = static_cast<uint8_t*>(workspace) + half;
  if (D == 64)
    return launch<64>(q, k, v, is_sep, prefix, idx, B, Hq, Hkv, S, a, n, scale, out, lse, kc, vc,
                      st);
  if (D == 128)
    return launch<128>(q, k, v, is_sep, prefix, idx, B, Hq, Hkv, S, a, n, scale, out, lse, kc, vc,
                       st);
  return SEP_EDTYPE;
}
}  // namespace sep
