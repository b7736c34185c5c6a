// Sep-Attention backward (bf16, D in {64, 128}): warp-level tensor cores
// (mma.sync) for D = 64, tcgen05 for D = 128 (second part of this file).
//
// Gradients of sum(out * dout) through the prefill's sparse attention (the
// training use of Sep-Attention: "HKUDS047: SepLLM ..." study, section on the
// three versions, Training-SepLLM; kept set of query i from section
// "SepAttention": {j <= i : j < a or is_sep[j] or i - j < n}).  Per kept pair
// (i, j), with p_ij the forward's probability (rebuilt from the saved lse)
// and delta_i = dout_i . out_i:
//   dv_j += p_ij dout_i,   ds_ij = p_ij (dout_i . v_j - delta_i),
//   dk_j += scale ds_ij q_i,   dq_i += scale ds_ij k_j.
//
// Key-centric work split.  The kept pairs fall into two disjoint families:
//   * global keys (j < a or a separator) are kept by every query i >= j;
//     they are taken 64 at a time from the separator index list, and each
//     block visits the query tiles after its first position, at most
//     kChunkTiles tiles per CTA;
//   * local keys (all others) are kept only by queries i in [j, j + n); they
//     are taken as 64 consecutive positions, and each block visits the query
//     tiles that reach it, with the global keys of the block masked out.
// A CTA (four warps, one work item) keeps its 64 keys' K and V in shared
// memory and the dK and dV of its keys in registers (warp w: keys 16w ..
// 16w + 15) over all query heads of the kv group and all its query tiles.
// Per 64-row query tile the warps form S^T = K Q^T and dP^T = V dO^T for
// their keys (the keys as the 16 rows of the mma tile), P and dS in
// registers, dV += P^T dO and dK += dS^T Q; dS goes to shared memory and each
// warp then forms dQ for 16 queries (dS K) and adds it into an fp32
// accumulator with vector reductions.  At the end the item adds its dK and
// dV into fp32 accumulators.  A delta pass runs before, and a pass after
// converts the accumulators (times scale for dq and dk) to bf16.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

constexpr int BR = 64;          // query rows per tile
constexpr int BC = 64;          // keys per work item
constexpr int kThreads = 128;   // four warps
constexpr int kChunkTiles = 4;  // query tiles per item of global keys (measured: 4 < 8 < 16)
constexpr int kTileBytes = 64 * 128;  // 64 rows x 64 bf16, 128-byte swizzled

// Byte offset of (row r, element d) in a tensor's D/64 swizzled 64-row tiles.
__device__ __forceinline__ uint32_t swz(int r, int d) {
  return static_cast<uint32_t>((d >> 6) * kTileBytes + r * 128 +
                               ((((d >> 3) & 7) ^ (r & 7)) << 4) + (d & 7) * 2);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// c (16x8 fp32) += a (16x16 bf16, row-major fragment) * b (16x8 bf16, col fragment)
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void red_add_v2(float* p, float x, float y) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(x), "f"(y) : "memory");
}

struct BwdParams {
  const __nv_bfloat16 *q, *k, *v, *dout;
  const float* lse;    // [B][Hq][S] natural log
  const float* delta;  // [B][Hq][S]
  const uint8_t* is_sep;
  const int32_t *prefix, *idx;
  float *dq_acc, *dk_acc, *dv_acc;
  int32_t* err;
  int B, Hq, Hkv, S, a, n;
  int nwin;     // window items per (b, kv head) = ceil(S / 64)
  int nchunk;   // chunks per block of global keys = ceil(ceil(S / 64) / kChunkTiles)
  float scale_log2;
};

// delta[b,h,i] = sum_d dout . out, one warp per row
template <int D>
__global__ void k_bwd_delta(const __nv_bfloat16* __restrict__ out,
                            const __nv_bfloat16* __restrict__ dout, float* __restrict__ delta,
                            int64_t rows) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int PER = D / 32;  // 2 or 4 elements per lane
  float acc = 0.f;
  const __nv_bfloat16* o = out + row * D + lane * PER;
  const __nv_bfloat16* g = dout + row * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) acc += __bfloat162float(o[e]) * __bfloat162float(g[e]);
#pragma unroll
  for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (lane == 0) delta[row] = acc;
}

// fp32 accumulators -> bf16 gradients (dq, dk scaled)
__global__ void k_bwd_convert(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dst,
                              int64_t n4, float mul) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float4 x = reinterpret_cast<const float4*>(acc)[i];
    __nv_bfloat162 lo = __floats2bfloat162_rn(x.x * mul, x.y * mul);
    __nv_bfloat162 hi = __floats2bfloat162_rn(x.z * mul, x.w * mul);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&lo);
    u.y = *reinterpret_cast<uint32_t*>(&hi);
    reinterpret_cast<uint2*>(dst)[i] = u;
  }
}

// Shared memory of one CTA (dynamic): K, V [64][D]; Q, dO [2][64][D]; dS^T
// [64 keys][64 queries], all bf16 swizzled; then the per-tile and per-key
// scalars.
template <int D>
struct Smem {
  static constexpr int T = (D / 64) * kTileBytes;  // one 64-row tensor
  static constexpr int K = 0, V = T, Q = 2 * T, DO = 4 * T, DS = 6 * T;
  static constexpr int LSE = DS + kTileBytes;      // [2][64] fp32 (log2 domain)
  static constexpr int DEL = LSE + 2 * 64 * 4;     // [2][64] fp32
  static constexpr int POS = DEL + 2 * 64 * 4;     // [64] int32 key positions
  static constexpr int LOCAL = POS + 64 * 4;       // [64] int32: key may be used
  static constexpr int BYTES = LOCAL + 64 * 4;
};

// D = 64 fits three CTAs per SM (registers <= 168), D = 128 two
template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 3 : 2) k_sep_bwd(const BwdParams p) {
  constexpr int DT = D / 16, NT = D / 8;
  using SM = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const uint32_t sbase = sep::smem_u32(smem);
  float* const lse_s = reinterpret_cast<float*>(smem + SM::LSE);
  float* const del_s = reinterpret_cast<float*>(smem + SM::DEL);
  int32_t* const pos_s = reinterpret_cast<int32_t*>(smem + SM::POS);
  int32_t* const use_s = reinterpret_cast<int32_t*>(smem + SM::LOCAL);

  const int item = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int S = p.S, G = p.Hq / p.Hkv;
  const int nT = (S + BR - 1) / BR;
  const int32_t* pre = p.prefix + static_cast<int64_t>(b) * (S + 1);
  const int32_t* ix = p.idx + static_cast<int64_t>(b) * S;
  const uint8_t* fl = p.is_sep + static_cast<int64_t>(b) * S;
  const int a0 = p.a < S ? p.a : S;
  const int nglob = a0 + (pre[S] - pre[a0]);  // global keys: initial, then separators >= a

  // ---- the item: its keys and its query tiles
  const bool window = item < p.nwin;
  int kb, t0, t1;
  if (window) {
    kb = item;
    t0 = kb;  // queries from the block's first key on
    const int last = kb * BC + BC - 1 + p.n - 1;  // the last query a key of the block can reach
    t1 = (last < S - 1 ? last : S - 1) / BR + 1;
  } else {
    kb = (item - p.nwin) / p.nchunk;
    const int chunk = (item - p.nwin) % p.nchunk;
    if (kb * BC >= nglob) return;
    const int t = kb * BC;
    const int pmin = t < a0 ? t : ix[pre[a0] + t - a0];
    t0 = pmin / BR + chunk * kChunkTiles;
    t1 = t0 + kChunkTiles < nT ? t0 + kChunkTiles : nT;
    if (t0 >= nT) return;
  }
  // key positions and whether a key takes part in this item's pairs
  if (threadIdx.x < BC) {
    const int r = threadIdx.x;
    int pos = -1, use = 0;
    if (window) {
      pos = kb * BC + r;
      use = pos < S && !(pos < p.a || fl[pos]);  // local keys only
      if (pos >= S) pos = -1;
    } else {
      const int t = kb * BC + r;
      if (t < nglob) {
        pos = t < a0 ? t : ix[pre[a0] + t - a0];
        use = 1;
      }
    }
    pos_s[r] = pos;
    use_s[r] = use;
  }
  __syncthreads();
  // K and V rows of the block (zero rows where there is no key)
  const int64_t kvrow0 = (static_cast<int64_t>(b) * p.Hkv + g) * S;
  for (int e = threadIdx.x; e < BC * (D / 8); e += kThreads) {
    const int r = e / (D / 8), c = e % (D / 8);
    const int pos = pos_s[r];
    const int64_t off = (kvrow0 + (pos < 0 ? 0 : pos)) * D + 8 * c;
    const uint32_t nb = pos < 0 ? 0u : 16u;
    cp_async16(sbase + SM::K + swz(r, 8 * c), p.k + off, nb);
    cp_async16(sbase + SM::V + swz(r, 8 * c), p.v + off, nb);
  }
  cp_async_commit();

  // the visits: (head, query tile) pairs, heads outer
  const int ntile = t1 - t0;
  const int nvisit = G * ntile;
  auto load_visit = [&](int v, int buf) {
    const int h = g * G + v / ntile, t = t0 + v % ntile;
    const int64_t qrow0 = (static_cast<int64_t>(b) * p.Hq + h) * S;
    for (int e = threadIdx.x; e < BR * (D / 8); e += kThreads) {
      const int r = e / (D / 8), c = e % (D / 8);
      const int i = t * BR + r;
      const int64_t off = (qrow0 + (i < S ? i : 0)) * D + 8 * c;
      const uint32_t nb = i < S ? 16u : 0u;
      cp_async16(sbase + SM::Q + buf * SM::T + swz(r, 8 * c), p.q + off, nb);
      cp_async16(sbase + SM::DO + buf * SM::T + swz(r, 8 * c), p.dout + off, nb);
    }
    if (threadIdx.x < BR) {
      const int i = t * BR + threadIdx.x;
      lse_s[buf * 64 + threadIdx.x] = i < S ? p.lse[qrow0 + i] * 1.44269504088896340736f : 0.f;
      del_s[buf * 64 + threadIdx.x] = i < S ? p.delta[qrow0 + i] : 0.f;
    }
    cp_async_commit();
  };
  if (nvisit > 0) load_visit(0, 0);

  float dk[NT][4], dv[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[nt][e] = dv[nt][e] = 0.f;

  const int kr = 16 * warp;  // this warp's keys
  for (int v = 0; v < nvisit; ++v) {
    const int buf = v & 1;
    const int h = g * G + v / ntile, t = t0 + v % ntile;
    const int i0 = t * BR;
    if (v + 1 < nvisit) {
      load_visit(v + 1, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this visit's tiles (and K, V) are in shared memory
    const uint32_t qs = sbase + SM::Q + buf * SM::T, ds_ = sbase + SM::DO + buf * SM::T;
    const uint32_t ks = sbase + SM::K, vs = sbase + SM::V, dss = sbase + SM::DS;
    const float* lse2 = lse_s + buf * 64;
    const float* del = del_s + buf * 64;
    // key rows of this lane: kr + gq and kr + gq + 8
    const int jp0 = pos_s[kr + gq], jp1 = pos_s[kr + gq + 8];
    const int u0 = use_s[kr + gq], u1 = use_s[kr + gq + 8];
    // the warp's last key position: a global-key item keeps every valid key
    // for queries after it, so those sub-blocks need no element mask
    int jmax = jp0 > jp1 ? jp0 : jp1;
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) jmax = max(jmax, __shfl_xor_sync(0xffffffffu, jmax, off));
    // ---------------- phase A: 16 queries at a time
#pragma unroll 1
    for (int sb = 0; sb < BR / 16; ++sb) {
      float s[2][4] = {}, dp[2][4] = {};
#pragma unroll
      for (int kk = 0; kk < DT; ++kk) {
        uint32_t ka[4], va[4], qb[4], ob[4];
        ldsm_x4(ks + swz(kr + (lane & 7) + ((lane >> 3) & 1) * 8, 16 * kk + (lane >> 4) * 8), ka);
        ldsm_x4(vs + swz(kr + (lane & 7) + ((lane >> 3) & 1) * 8, 16 * kk + (lane >> 4) * 8), va);
        // B = Q^T / dO^T: matrices (queries 0-7 | 8-15) x (dims 16kk | 16kk+8)
        const int qr = 16 * sb + (lane & 7) + (lane >> 4) * 8, qc = 16 * kk + ((lane >> 3) & 1) * 8;
        ldsm_x4(qs + swz(qr, qc), qb);
        ldsm_x4(ds_ + swz(qr, qc), ob);
        mma16816(s[0], ka, qb[0], qb[1]);
        mma16816(s[1], ka, qb[2], qb[3]);
        mma16816(dp[0], va, ob[0], ob[1]);
        mma16816(dp[1], va, ob[2], ob[3]);
      }
      // P and dS: element e of n-tile nt is key kr + gq (+8 for e >= 2),
      // query 16sb + 8nt + 2tq + (e & 1)
      uint32_t pa[4], sa[4];
      // (D = 128 runs at the register limit, where the extra path costs more
      // than it saves: measured)
      const bool all_kept = D == 64 && !window && i0 + 16 * sb >= jmax && i0 + 16 * sb + 15 < S;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        float pv[4], dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = 16 * sb + 8 * nt + 2 * tq + (e & 1);
          const int i = i0 + q;
          const int j = e < 2 ? jp0 : jp1;
          const int use = e < 2 ? u0 : u1;
          bool kept;
          if (all_kept) {
            kept = use;
          } else {
            kept = use && j >= 0 && i < S && j <= i;
            if (window) kept = kept && i - j < p.n;
          }
          const float pe = kept ? exp2f(s[nt][e] * p.scale_log2 - lse2[q]) : 0.f;
          pv[e] = pe;
          dsv[e] = pe * (dp[nt][e] - del[q]);
        }
        pa[2 * nt] = sep::pack_bf16x2(pv[0], pv[1]);
        pa[2 * nt + 1] = sep::pack_bf16x2(pv[2], pv[3]);
        sa[2 * nt] = sep::pack_bf16x2(dsv[0], dsv[1]);
        sa[2 * nt + 1] = sep::pack_bf16x2(dsv[2], dsv[3]);
        // dS^T to shared memory: rows keys, columns queries
        const int q0 = 16 * sb + 8 * nt + 2 * tq;
        *reinterpret_cast<uint32_t*>(smem + SM::DS + swz(kr + gq, q0)) = sa[2 * nt];
        *reinterpret_cast<uint32_t*>(smem + SM::DS + swz(kr + gq + 8, q0)) = sa[2 * nt + 1];
      }
      // A fragments of P^T / dS^T (keys x 16 queries): registers 0, 1 of
      // n-tile 0 and 0, 1 of n-tile 1
      const uint32_t ap[4] = {pa[0], pa[1], pa[2], pa[3]};
      const uint32_t as[4] = {sa[0], sa[1], sa[2], sa[3]};
      // dV += P^T dO, dK += dS^T Q: B = dO / Q (queries x dims) by ldmatrix.trans
#pragma unroll
      for (int dn = 0; dn < NT; dn += 2) {
        uint32_t ob[4], qb[4];
        const int rr = 16 * sb + (lane & 7) + ((lane >> 3) & 1) * 8, cc = 8 * dn + (lane >> 4) * 8;
        ldsm_x4_t(ds_ + swz(rr, cc), ob);
        ldsm_x4_t(qs + swz(rr, cc), qb);
        mma16816(dv[dn], ap, ob[0], ob[1]);
        mma16816(dv[dn + 1], ap, ob[2], ob[3]);
        mma16816(dk[dn], as, qb[0], qb[1]);
        mma16816(dk[dn + 1], as, qb[2], qb[3]);
      }
    }
    __syncthreads();  // dS^T of all keys is in shared memory
    // ---------------- phase B: dQ of queries 16w .. 16w + 15 = dS K, one
    // half of the dims at a time (half the accumulator registers)
    {
      const int64_t qrow0 = (static_cast<int64_t>(b) * p.Hq + h) * S;
#pragma unroll 1
      for (int dh = 0; dh < 2; ++dh) {
        float dq[NT / 2][4];
#pragma unroll
        for (int nt = 0; nt < NT / 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
#pragma unroll
        for (int kt = 0; kt < BC / 16; ++kt) {
          // A = dS (queries x keys) from dS^T by ldmatrix.trans: matrices
          // (keys 16kt | +8) x (queries 16w | +8)
          uint32_t aa[4];
          {
            const int m = lane >> 3, r = lane & 7;
            const int key = 16 * kt + (m >> 1) * 8 + r, q = 16 * warp + (m & 1) * 8;
            ldsm_x4_t(dss + swz(key, q), aa);
          }
#pragma unroll
          for (int dn = 0; dn < NT / 2; dn += 2) {
            // B = K (keys x dims) by ldmatrix.trans: matrices (keys | +8) x (dims | +8)
            uint32_t kb4[4];
            const int m = lane >> 3, r = lane & 7;
            const int key = 16 * kt + (m & 1) * 8 + r, d = 8 * (dh * (NT / 2) + dn) + (m >> 1) * 8;
            ldsm_x4_t(ks + swz(key, d), kb4);
            mma16816(dq[dn], aa, kb4[0], kb4[1]);
            mma16816(dq[dn + 1], aa, kb4[2], kb4[3]);
          }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int i = i0 + 16 * warp + gq + 8 * half;
          if (i < S) {
            float* dst = p.dq_acc + (qrow0 + i) * D + (D / 2) * dh + 2 * tq;
#pragma unroll
            for (int nt = 0; nt < NT / 2; ++nt) red_add_v2(dst + 8 * nt, dq[nt][2 * half], dq[nt][2 * half + 1]);
          }
        }
      }
    }
    __syncthreads();  // the buffers of this visit may be refilled
  }
  // ---------------- the item's dK and dV
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int key = kr + gq + 8 * half;
    const int j = pos_s[key];
    if (j >= 0 && use_s[key]) {
      float* dkp = p.dk_acc + (kvrow0 + j) * D + 2 * tq;
      float* dvp = p.dv_acc + (kvrow0 + j) * D + 2 * tq;
      if (window) {  // a local key's pairs all belong to this item: plain stores
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          *reinterpret_cast<float2*>(dkp + 8 * nt) = make_float2(dk[nt][2 * half], dk[nt][2 * half + 1]);
          *reinterpret_cast<float2*>(dvp + 8 * nt) = make_float2(dv[nt][2 * half], dv[nt][2 * half + 1]);
        }
      } else {  // global keys: one item per chunk of query tiles
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          red_add_v2(dkp + 8 * nt, dk[nt][2 * half], dk[nt][2 * half + 1]);
          red_add_v2(dvp + 8 * nt, dv[nt][2 * half], dv[nt][2 * half + 1]);
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// tcgen05 form (D = 128), two kernels on the operand forms of the forward:
//   k_sep_bwd_tc_kv (key-centric, 128 keys in TMEM lanes, 128-query tiles,
//     Q and dO double-buffered): S^T = K Q^T and dP^T = V dO^T (SS); warps
//     0-3 (thread = key row) turn them into P^T and dS^T, written back as
//     bf16 over the first 64 columns of each; dV += P^T dO and dK += dS^T Q
//     (TS, B MN-major).  TMEM: S^T [0,128) dP^T [128,256) dV [256,384)
//     dK [384,512).
//   k_sep_bwd_tc_q (query-centric, 128 queries in TMEM lanes, over the kept
//     key blocks of its tile as the forward does: the global keys before the
//     window unmasked, then the window blocks with the element mask; K and V
//     double-buffered): S = Q K^T and dP = dO V^T (SS); thread = query row
//     forms dS, written back as bf16; dQ += dS K (TS, B = K MN-major).  The
//     CTA owns its queries, so dQ is stored once, as bf16, with no
//     reduction.  TMEM: S [0,128) dP [128,256) dQ [256,384).
// Warps 0-7 share the 128 TMEM lanes two by two (warp w: lanes 32 (w & 3) ..
// +31, columns [64 (w >> 2), +64) of each 128-column tile); the two warps of
// a lane quarter load all their scores before either stores the bf16 P / dS
// over them.  Warp 8 allocates TMEM; its lane 0 issues the MMAs (and, in the
// key-centric kernel, the tensor copies of the Q and dO tiles) while the
// other lanes wait for it, and the warp reaches the block barrier together.
constexpr int TBK = 128;  // keys per block (TMEM lanes of the key-centric kernel)
constexpr int TBQ = 128;  // queries per tile
constexpr int kTcThreads = 288;  // warps 0-7: softmax, loads, readout; warp 8: TMEM and MMA issue
constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDQ = 256;
template <int D>
constexpr uint32_t col_dk() { return kColDV + D; }  // dK after the D columns of dV
constexpr int kT128 = 128 * 128;  // one 128-row x 64-column swizzled tile
constexpr int kTcChunkTiles = 4;  // query tiles per item of global keys

__device__ __forceinline__ uint32_t swz128(int r, int d) {
  return static_cast<uint32_t>((d >> 6) * kT128 + r * 128 + ((((d >> 3) & 7) ^ (r & 7)) << 4) +
                               (d & 7) * 2);
}
// packed fp32 pairs (one f32x2 instruction per pair)
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "sub.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// kind::f16 instruction descriptor with bf16 A/B, fp32 D and each operand's
// major-ness (bit 15: A MN-major, bit 16: B MN-major)
__host__ __device__ constexpr uint32_t idesc_mn(int M, int N, bool a_mn, bool b_mn) {
  return sep::idesc_bf16_f32(M, N, b_mn) | ((a_mn ? 1u : 0u) << 15);
}
// Rows [0, 128) of a [rows, D] bf16 tensor into D/64 swizzled 128-row
// tiles, one 16-byte chunk per copy; row_of(r) < 0 gives a zero row.
template <int D, typename RowOf>
__device__ __forceinline__ void load_rows(uint32_t dst, const __nv_bfloat16* src, RowOf row_of,
                                          int tid, int nthreads) {
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int e = tid; e < 128 * CH; e += nthreads) {
    const int r = e / CH, c = e % CH;
    const int64_t row = row_of(r);
    cp_async16(dst + swz128(r, 8 * c), src + (row < 0 ? 0 : row) * D + 8 * c, row < 0 ? 0u : 16u);
  }
}

// NB = D/64 tiles of 128 rows x 64 columns per 128-row tensor
template <int D>
struct KvSmem {
  static constexpr int NB = D / 64;
  static constexpr int K = 0, V = NB * kT128, Q = 2 * NB * kT128, DO = 4 * NB * kT128;  // Q, dO: [2] x NB tiles
  static constexpr int LSE = 6 * NB * kT128;  // [2][128] fp32: -lse (log2 domain)
  static constexpr int DEL = LSE + 1024;  // [2][128] fp32
  static constexpr int POS = DEL + 1024;  // [128] int32
  static constexpr int USE = POS + 512;   // [128] int32
  static constexpr int BYTES = USE + 512 + 1024;  // + alignment slack
};
struct TcBars {
  uint64_t full, s_full, p_full, m_full, drain;
  uint64_t tile[2];  // tensor-copy completion of a Q / dO buffer (key-centric kernel)
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_sep_bwd_tc_kv(const BwdParams p, const __grid_constant__ CUtensorMap map_q,
                    const __grid_constant__ CUtensorMap map_do) {
  using KvSmem = ::KvSmem<D>;
  constexpr int NB = D / 64;
  constexpr uint32_t kColDK = col_dk<D>();
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* const smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ TcBars bars;
  const uint32_t sb_ = sep::smem_u32(smem);
  float* const lse_s = reinterpret_cast<float*>(smem + KvSmem::LSE);
  float* const del_s = reinterpret_cast<float*>(smem + KvSmem::DEL);
  int32_t* const pos_s = reinterpret_cast<int32_t*>(smem + KvSmem::POS);
  int32_t* const use_s = reinterpret_cast<int32_t*>(smem + KvSmem::USE);

  const int item = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, G = p.Hq / p.Hkv;
  const int nT = (S + TBQ - 1) / TBQ;
  const int32_t* pre = p.prefix + static_cast<int64_t>(b) * (S + 1);
  const int32_t* ix = p.idx + static_cast<int64_t>(b) * S;
  const uint8_t* fl = p.is_sep + static_cast<int64_t>(b) * S;
  const int a0 = p.a < S ? p.a : S;
  const int nglob = a0 + (pre[S] - pre[a0]);

  const bool window = item < p.nwin;
  int kb, t0, t1;
  if (window) {
    kb = item;
    t0 = kb;
    const int last = kb * TBK + TBK - 1 + p.n - 1;
    t1 = (last < S - 1 ? last : S - 1) / TBQ + 1;
  } else {
    kb = (item - p.nwin) / p.nchunk;
    const int chunk = (item - p.nwin) % p.nchunk;
    if (kb * TBK >= nglob) return;
    const int t = kb * TBK;
    const int pmin = t < a0 ? t : ix[pre[a0] + t - a0];
    t0 = pmin / TBQ + chunk * kTcChunkTiles;
    t1 = t0 + kTcChunkTiles < nT ? t0 + kTcChunkTiles : nT;
    if (t0 >= nT) return;
  }
  const int ntile = t1 - t0;
  const int nvisit = G * ntile;

  if (threadIdx.x == 0) {
    sep::mbar_init(&bars.full, 1);
    sep::mbar_init(&bars.s_full, 1);
    sep::mbar_init(&bars.p_full, 1);
    sep::mbar_init(&bars.m_full, 1);
    sep::mbar_init(&bars.drain, 1);
    sep::mbar_init(&bars.tile[0], 1);
    sep::mbar_init(&bars.tile[1], 1);
    bars.abort = 0;
    sep::mbar_fence_init();
  }
  if (threadIdx.x < TBK) {
    const int r = threadIdx.x;
    int pos = -1, use = 0;
    if (window) {
      pos = kb * TBK + r;
      use = pos < S && !(pos < p.a || fl[pos]);
      if (pos >= S) pos = -1;
    } else {
      const int t = kb * TBK + r;
      if (t < nglob) {
        pos = t < a0 ? t : ix[pre[a0] + t - a0];
        use = 1;
      }
    }
    pos_s[r] = pos;
    use_s[r] = use;
  }
  if (warp == 8) {
    sep::tmem_alloc(&bars.tmem_base, 512);
    sep::tmem_relinquish();
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  volatile int* abort = &bars.abort;
  const int64_t kvrow0 = (static_cast<int64_t>(b) * p.Hkv + g) * S;

  if (warp < 8) {
    // ------------------------------------------------ compute warps
    const int tid = threadIdx.x;
    const int lq = warp & 3, ch = warp >> 2;
    const int r = 32 * lq + lane;  // key row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * lq) << 16;
    load_rows<D>(sb_ + KvSmem::K, p.k, [&](int rr) { const int q = pos_s[rr]; return q < 0 ? -1 : kvrow0 + q; }, tid, 256);
    load_rows<D>(sb_ + KvSmem::V, p.v, [&](int rr) { const int q = pos_s[rr]; return q < 0 ? -1 : kvrow0 + q; }, tid, 256);
    cp_async_commit();
    // lse (negated, log2 domain) and delta of visit v's queries: thread
    // tid < 128 loads its query's pair (into registers one visit ahead)
    auto row_stats = [&](int v, float& nl, float& dl) {
      const int h = g * G + v / ntile, t = t0 + v % ntile;
      const int i = t * TBQ + tid;
      const int64_t qrow0 = (static_cast<int64_t>(b) * p.Hq + h) * S;
      nl = i < S ? -p.lse[qrow0 + i] * 1.44269504088896340736f : 0.f;
      dl = i < S ? p.delta[qrow0 + i] : 0.f;
    };
    if (tid < TBQ) {
      float nl, dl;
      row_stats(0, nl, dl);
      lse_s[tid] = nl;
      del_s[tid] = dl;
    }
    cp_async_wait<0>();  // K and V
    sep::fence_proxy_async_smem();
    sep::named_bar_sync(1, 256);
    if (tid == 0) sep::mbar_arrive(&bars.full);  // K and V are in shared memory
    const int jp = pos_s[r], use = use_s[r];
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    bool ok = true;
    for (int v = 0; v < nvisit && ok; ++v) {
      const int buf = v & 1;
      const int t = t0 + v % ntile;
      const int i0 = t * TBQ;
      float nl_next = 0.f, dl_next = 0.f;
      if (v + 1 < nvisit && tid < TBQ) row_stats(v + 1, nl_next, dl_next);
      if (!sep::mbar_wait(&bars.s_full, v & 1, abort, p.err) || *abort) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      // the query columns this key row keeps: [qa, qb)
      int qa = 0, qb = 0;
      if (use && jp >= 0) {
        qa = jp - i0 > 0 ? jp - i0 : 0;
        qb = S - i0 < TBQ ? S - i0 : TBQ;
        if (window && jp + p.n - i0 < qb) qb = jp + p.n - i0;
      }
      uint32_t sv[64], dv_[64];
      sep::tmem_ld32(tmem + lane_base + kColS + 64 * ch, sv);
      sep::tmem_ld32(tmem + lane_base + kColS + 64 * ch + 32, sv + 32);
      sep::tmem_ld32(tmem + lane_base + kColDP + 64 * ch, dv_);
      sep::tmem_ld32(tmem + lane_base + kColDP + 64 * ch + 32, dv_ + 32);
      sep::tmem_wait_ld_r32(sv);
      sep::tmem_wait_ld_r32(sv + 32);
      sep::tmem_wait_ld_r32(dv_);
      sep::tmem_wait_ld_r32(dv_ + 32);
      sep::named_bar_sync(2 + lq, 64);  // the partner warp has read its scores too
      const float* nl = lse_s + buf * 128 + 64 * ch;
      const float* dl = del_s + buf * 128 + 64 * ch;
      uint32_t pp[32], dd[32];
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        const int q = 64 * ch + e;
        const float2 x = sep::ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2,
                                    *reinterpret_cast<const float2*>(nl + e));
        const float p0 = (q >= qa && q < qb) ? sep::ex2_approx(x.x) : 0.f;
        const float p1 = (q + 1 >= qa && q + 1 < qb) ? sep::ex2_approx(x.y) : 0.f;
        const float2 ds = fmul2(make_float2(p0, p1),
                                fsub2(make_float2(__uint_as_float(dv_[e]), __uint_as_float(dv_[e + 1])),
                                      *reinterpret_cast<const float2*>(dl + e)));
        pp[e / 2] = sep::pack_bf16x2(p0, p1);
        dd[e / 2] = sep::pack_bf16x2(ds.x, ds.y);
      }
      sep::tmem_st32(tmem + lane_base + kColS + 32 * ch, pp);
      sep::tmem_st32(tmem + lane_base + kColDP + 32 * ch, dd);
      if (v + 1 < nvisit && tid < TBQ) {  // buffer (v+1) & 1 was last read by visit v-1
        lse_s[(buf ^ 1) * 128 + tid] = nl_next;
        del_s[(buf ^ 1) * 128 + tid] = dl_next;
      }
      sep::tmem_wait_st();
      sep::tc_fence_before();
      sep::named_bar_sync(1, 256);
      if (tid == 0) sep::mbar_arrive(&bars.p_full);
    }
    if (ok && nvisit > 0 && sep::mbar_wait(&bars.m_full, (nvisit - 1) & 1, abort, p.err) && !*abort) {
      sep::tc_fence_after();
      // dK and dV of this key row, columns [D/2 ch, +D/2): every lane
      // loads (warp-wide), rows with a key store
      const bool mine = jp >= 0 && use;
      float* dkp = p.dk_acc + (kvrow0 + (mine ? jp : 0)) * D + (D / 2) * ch;
      float* dvp = p.dv_acc + (kvrow0 + (mine ? jp : 0)) * D + (D / 2) * ch;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t kv[32], vv[32];
        sep::tmem_ld32(tmem + lane_base + kColDK + (D / 2) * ch + 32 * c, kv);
        sep::tmem_ld32(tmem + lane_base + kColDV + (D / 2) * ch + 32 * c, vv);
        sep::tmem_wait_ld_r32(kv);
        sep::tmem_wait_ld_r32(vv);
        if (mine) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            if (window) {
              *reinterpret_cast<float2*>(dkp + 32 * c + e) = make_float2(__uint_as_float(kv[e]), __uint_as_float(kv[e + 1]));
              *reinterpret_cast<float2*>(dvp + 32 * c + e) = make_float2(__uint_as_float(vv[e]), __uint_as_float(vv[e + 1]));
            } else {
              red_add_v2(dkp + 32 * c + e, __uint_as_float(kv[e]), __uint_as_float(kv[e + 1]));
              red_add_v2(dvp + 32 * c + e, __uint_as_float(vv[e]), __uint_as_float(vv[e + 1]));
            }
          }
        }
      }
    }
    cp_async_wait<0>();
  } else {
    if (lane == 0) {
      // ---------------------------------------------- MMA issue (one thread)
      constexpr uint32_t id_s = idesc_mn(128, 128, false, false);
      constexpr uint32_t id_o = idesc_mn(128, D, false, true);
      const uint64_t dK = sep::smem_desc_sw128(sb_ + KvSmem::K, 16);
      const uint64_t dV = sep::smem_desc_sw128(sb_ + KvSmem::V, 16);
      // Q and dO tiles of visit v into buffer v & 1 by the tensor-copy
      // engine (two 64-column tiles each; rows past the head belong to the
      // next head or are zero-filled past the array, and their P is 0)
      auto load_tiles = [&](int v) {
        const int h = g * G + v / ntile, t = t0 + v % ntile;
        const int32_t row = static_cast<int32_t>((static_cast<int64_t>(b) * p.Hq + h) * S + t * TBQ);
        const int buf = v & 1;
        sep::mbar_arrive_expect_tx(&bars.tile[buf], 2 * NB * kT128);
#pragma unroll
        for (int c = 0; c < NB; ++c) {
          sep::tma_load_2d(smem + KvSmem::Q + buf * NB * kT128 + c * kT128, &map_q, 64 * c, row, &bars.tile[buf]);
          sep::tma_load_2d(smem + KvSmem::DO + buf * NB * kT128 + c * kT128, &map_do, 64 * c, row, &bars.tile[buf]);
        }
      };
      if (nvisit > 0) load_tiles(0);
      bool kv_in = sep::mbar_wait(&bars.full, 0, abort, p.err);  // K and V
      for (int v = 0; v < nvisit && kv_in; ++v) {
        const int buf = v & 1;
        if (!sep::mbar_wait(&bars.tile[buf], (v >> 1) & 1, abort, p.err)) break;
        sep::tc_fence_after();
        const uint32_t qa = sb_ + KvSmem::Q + buf * NB * kT128, oa = sb_ + KvSmem::DO + buf * NB * kT128;
        const uint64_t dQ = sep::smem_desc_sw128(qa, 16), dO = sep::smem_desc_sw128(oa, 16);
        const uint64_t dQmn = sep::smem_desc_sw128(qa, kT128), dOmn = sep::smem_desc_sw128(oa, kT128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * kT128 + (kk % 4) * 32) >> 4);
          sep::mma_bf16_ss(tmem + kColS, dK + off, dQ + off, id_s, kk > 0 ? 1u : 0u);
          sep::mma_bf16_ss(tmem + kColDP, dV + off, dO + off, id_s, kk > 0 ? 1u : 0u);
        }
        sep::mma_commit(&bars.s_full);
        if (!sep::mbar_wait(&bars.p_full, v & 1, abort, p.err)) break;
        // the scores of visit v are complete, so (in order) are the products
        // of visit v-1: buffer (v+1) & 1 may be refilled
        if (v + 1 < nvisit) load_tiles(v + 1);
        sep::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TBQ / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(kk * (2048 >> 4));
          const uint32_t acc = (v > 0 || kk > 0) ? 1u : 0u;
          sep::mma_bf16_ts(tmem + kColDV, tmem + kColS + kk * 8, dOmn + off, id_o, acc);
          sep::mma_bf16_ts(tmem + kColDK, tmem + kColDP + kk * 8, dQmn + off, id_o, acc);
        }
        sep::mma_commit(&bars.m_full);
      }
      sep::mma_commit(&bars.drain);  // every MMA completes before TMEM is released
      int keep = 0;
      sep::mbar_wait(&bars.drain, 0, &keep, nullptr);
    }
    __syncwarp();
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  if (warp == 8) {
    __syncwarp();
    sep::tmem_dealloc(tmem, 512);
  }
}

template <int D>
struct QSmem {
  static constexpr int NB = D / 64;
  static constexpr int Q = 0, DO = NB * kT128;
  static constexpr int K = 2 * NB * kT128, V = 3 * NB * kT128;  // [2] buffers, 2 NB tiles apart
  static constexpr int POS = 6 * NB * kT128;  // [2][128] int32 key positions
  static constexpr int GLB = POS + 1024;  // [2][128] int32: key kept by every later query
  static constexpr int BYTES = GLB + 1024 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) k_sep_bwd_tc_q(const BwdParams p,
                                                                __nv_bfloat16* __restrict__ dq) {
  using QSmem = ::QSmem<D>;
  constexpr int NB = D / 64;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* const smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ TcBars bars;
  const uint32_t sb_ = sep::smem_u32(smem);
  int32_t* const pos_s = reinterpret_cast<int32_t*>(smem + QSmem::POS);
  int32_t* const glb_s = reinterpret_cast<int32_t*>(smem + QSmem::GLB);

  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, G = p.Hq / p.Hkv, g = h / G;
  const int i0 = t * TBQ;
  const int qlast = (i0 + TBQ < S ? i0 + TBQ : S) - 1;
  const int32_t* pre = p.prefix + static_cast<int64_t>(b) * (S + 1);
  const int32_t* ix = p.idx + static_cast<int64_t>(b) * S;
  const uint8_t* fl = p.is_sep + static_cast<int64_t>(b) * S;
  // the tile's kept keys: global keys before the first row's window, then
  // the window positions [lo, qlast]
  const int lo = i0 - p.n + 1 > 0 ? i0 - p.n + 1 : 0;
  const int al = p.a < lo ? p.a : lo;
  const int nglo = al + (pre[lo] - pre[al]);
  const int nbg = (nglo + TBK - 1) / TBK;
  const int nbw = (qlast - lo + TBK) / TBK;
  const int nblk = nbg + nbw;
  const int64_t kvrow0 = (static_cast<int64_t>(b) * p.Hkv + g) * S;
  const int64_t qrow0 = (static_cast<int64_t>(b) * p.Hq + h) * S;

  if (threadIdx.x == 0) {
    sep::mbar_init(&bars.full, 1);
    sep::mbar_init(&bars.s_full, 1);
    sep::mbar_init(&bars.p_full, 1);
    sep::mbar_init(&bars.m_full, 1);
    sep::mbar_init(&bars.drain, 1);
    bars.abort = 0;
    sep::mbar_fence_init();
  }
  if (warp == 8) {
    sep::tmem_alloc(&bars.tmem_base, 512);
    sep::tmem_relinquish();
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  volatile int* abort = &bars.abort;

  if (warp < 8) {
    const int tid = threadIdx.x;
    const int lq = warp & 3, ch = warp >> 2;
    const int r = 32 * lq + lane;  // query row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * lq) << 16;
    const int i = i0 + r;
    const float nlse2 = i < S ? -p.lse[qrow0 + i] * 1.44269504088896340736f : 0.f;
    const float dl = i < S ? p.delta[qrow0 + i] : 0.f;
    auto rowq = [&](int rr) -> int64_t { return i0 + rr < S ? qrow0 + i0 + rr : -1; };
    load_rows<D>(sb_ + QSmem::Q, p.q, rowq, tid, 256);
    load_rows<D>(sb_ + QSmem::DO, p.dout, rowq, tid, 256);
    auto load_block = [&](int j, int buf) {
      // key positions of block j (threads 0..127: one key each), then rows
      if (tid < TBK) {
        int pos = -1, glb = 0;
        if (j < nbg) {
          const int e = j * TBK + tid;
          if (e < nglo) {
            pos = e < al ? e : ix[pre[al] + e - al];
            glb = 1;
          }
        } else {
          const int q = lo + (j - nbg) * TBK + tid;
          if (q <= qlast) {
            pos = q;
            glb = q < p.a || fl[q];
          }
        }
        pos_s[buf * 128 + tid] = pos;
        glb_s[buf * 128 + tid] = glb;
      }
      sep::named_bar_sync(1, 256);  // every position is written before the row copies read them
      auto rowk = [&](int rr) -> int64_t { const int q = pos_s[buf * 128 + rr]; return q < 0 ? -1 : kvrow0 + q; };
      load_rows<D>(sb_ + QSmem::K + buf * 2 * NB * kT128, p.k, rowk, tid, 256);
      load_rows<D>(sb_ + QSmem::V + buf * 2 * NB * kT128, p.v, rowk, tid, 256);
      cp_async_commit();
    };
    load_block(0, 0);  // with Q and dO
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const float2 nl2 = make_float2(nlse2, nlse2), dl2 = make_float2(dl, dl);
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      const int buf = j & 1;
      if (j > 0 && (!sep::mbar_wait(&bars.m_full, (j - 1) & 1, abort, p.err) || *abort)) {
        ok = false;  // the products of block j-1 have read buffer (j+1) & 1
        break;
      }
      if (j + 1 < nblk) {
        load_block(j + 1, buf ^ 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      sep::fence_proxy_async_smem();
      sep::named_bar_sync(1, 256);
      if (tid == 0) sep::mbar_arrive(&bars.full);
      if (!sep::mbar_wait(&bars.s_full, j & 1, abort, p.err) || *abort) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      const int32_t* gb = glb_s + buf * 128 + 64 * ch;
      // the key columns this query row keeps: global blocks, every valid
      // key; window blocks (contiguous positions from `base`), keys at most
      // n - 1 back, or global ones, never past the row or the tile
      int ka, kb2;
      const bool win = j >= nbg;
      int wlo = 0;
      if (!win) {
        ka = 0;
        kb2 = nglo - j * TBK < TBK ? nglo - j * TBK : TBK;
        if (i >= S) kb2 = 0;
      } else {
        const int base = lo + (j - nbg) * TBK;
        ka = 0;
        kb2 = i - base + 1;  // keys at positions <= i
        const int lim = qlast - base + 1;
        if (kb2 > lim) kb2 = lim;
        if (kb2 > TBK) kb2 = TBK;
        if (i >= S) kb2 = 0;
        wlo = i - base - p.n + 1;  // keys before this column need the global flag
      }
      uint32_t sv[64], dv_[64];
      sep::tmem_ld32(tmem + lane_base + kColS + 64 * ch, sv);
      sep::tmem_ld32(tmem + lane_base + kColS + 64 * ch + 32, sv + 32);
      sep::tmem_ld32(tmem + lane_base + kColDP + 64 * ch, dv_);
      sep::tmem_ld32(tmem + lane_base + kColDP + 64 * ch + 32, dv_ + 32);
      sep::tmem_wait_ld_r32(sv);
      sep::tmem_wait_ld_r32(sv + 32);
      sep::tmem_wait_ld_r32(dv_);
      sep::tmem_wait_ld_r32(dv_ + 32);
      sep::named_bar_sync(2 + lq, 64);  // the partner warp has read its scores too
      uint32_t dd[32];
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        const int kc = 64 * ch + e;
        const float2 x = sep::ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), sc2, nl2);
        bool k0 = kc >= ka && kc < kb2, k1 = kc + 1 >= ka && kc + 1 < kb2;
        if (win) {
          k0 = k0 && (kc >= wlo || gb[e]);
          k1 = k1 && (kc + 1 >= wlo || gb[e + 1]);
        }
        const float p0 = k0 ? sep::ex2_approx(x.x) : 0.f;
        const float p1 = k1 ? sep::ex2_approx(x.y) : 0.f;
        const float2 ds = fmul2(make_float2(p0, p1),
                                fsub2(make_float2(__uint_as_float(dv_[e]), __uint_as_float(dv_[e + 1])), dl2));
        dd[e / 2] = sep::pack_bf16x2(ds.x, ds.y);
      }
      sep::tmem_st32(tmem + lane_base + kColS + 32 * ch, dd);
      sep::tmem_wait_st();
      sep::tc_fence_before();
      sep::named_bar_sync(1, 256);
      if (tid == 0) sep::mbar_arrive(&bars.p_full);
    }
    if (ok && sep::mbar_wait(&bars.m_full, (nblk - 1) & 1, abort, p.err) && !*abort) {
      sep::tc_fence_after();
      const float sc = p.scale_log2 * 0.69314718055994530942f;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t qv[32];
        sep::tmem_ld32(tmem + lane_base + kColDQ + (D / 2) * ch + 32 * c, qv);
        sep::tmem_wait_ld_r32(qv);
        if (i < S) {
          uint4* dst = reinterpret_cast<uint4*>(dq + (qrow0 + i) * D + (D / 2) * ch + 32 * c);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dst[u] = make_uint4(sep::pack_bf16x2(__uint_as_float(qv[8 * u]) * sc, __uint_as_float(qv[8 * u + 1]) * sc),
                                sep::pack_bf16x2(__uint_as_float(qv[8 * u + 2]) * sc, __uint_as_float(qv[8 * u + 3]) * sc),
                                sep::pack_bf16x2(__uint_as_float(qv[8 * u + 4]) * sc, __uint_as_float(qv[8 * u + 5]) * sc),
                                sep::pack_bf16x2(__uint_as_float(qv[8 * u + 6]) * sc, __uint_as_float(qv[8 * u + 7]) * sc));
        }
      }
    }
    cp_async_wait<0>();
  } else {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_mn(128, 128, false, false);
      constexpr uint32_t id_o = idesc_mn(128, D, false, true);
      const uint64_t dQ = sep::smem_desc_sw128(sb_ + QSmem::Q, 16);
      const uint64_t dO = sep::smem_desc_sw128(sb_ + QSmem::DO, 16);
      for (int j = 0; j < nblk; ++j) {
        const int buf = j & 1;
        if (!sep::mbar_wait(&bars.full, j & 1, abort, p.err)) break;
        sep::tc_fence_after();
        const uint32_t ka = sb_ + QSmem::K + buf * 2 * NB * kT128, va = sb_ + QSmem::V + buf * 2 * NB * kT128;
        const uint64_t dK = sep::smem_desc_sw128(ka, 16), dV = sep::smem_desc_sw128(va, 16);
        const uint64_t dKmn = sep::smem_desc_sw128(ka, kT128);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * kT128 + (kk % 4) * 32) >> 4);
          sep::mma_bf16_ss(tmem + kColS, dQ + off, dK + off, id_s, kk > 0 ? 1u : 0u);
          sep::mma_bf16_ss(tmem + kColDP, dO + off, dV + off, id_s, kk > 0 ? 1u : 0u);
        }
        sep::mma_commit(&bars.s_full);
        if (!sep::mbar_wait(&bars.p_full, j & 1, abort, p.err)) break;
        sep::tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TBK / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(kk * (2048 >> 4));
          sep::mma_bf16_ts(tmem + kColDQ, tmem + kColS + kk * 8, dKmn + off, id_o,
                           (j > 0 || kk > 0) ? 1u : 0u);
        }
        sep::mma_commit(&bars.m_full);
      }
      sep::mma_commit(&bars.drain);
      int keep = 0;
      sep::mbar_wait(&bars.drain, 0, &keep, nullptr);
    }
    __syncwarp();
  }
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  if (warp == 8) {
    __syncwarp();
    sep::tmem_dealloc(tmem, 512);
  }
}

// D = 128 runs the tcgen05 kernels.  At D = 64 they are correct too (the
// same kernels with one 64-column tile per 128-row tensor) but slower than
// the warp-level kernel on the Pythia-160M shape (0.54 against 0.37 ms per
// step): TMEM holds one CTA per SM and the items there are small.
template <int D>
constexpr bool tc_backward() { return D == 128; }

struct BwdWs {
  size_t delta, dq, dk, dv;
};
BwdWs bwd_ws(int B, int Hq, int Hkv, int S, int D) {
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  BwdWs w;
  w.delta = r256(static_cast<size_t>(B) * Hq * S * 4);
  w.dq = r256(static_cast<size_t>(B) * Hq * S * D * 4);
  w.dk = r256(static_cast<size_t>(B) * Hkv * S * D * 4);
  w.dv = w.dk;
  return w;
}

// the tcgen05 kernels: dK, dV key-centric; dQ query-centric
template <int D>
int launch_bwd_tc(BwdParams p, void* dq, cudaStream_t st) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(k_sep_bwd_tc_kv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             KvSmem<D>::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(k_sep_bwd_tc_q<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QSmem<D>::BYTES) != cudaSuccess)
      return SEP_ECUDA;
    attr_done[dev] = true;
  }
  p.nwin = (p.S + TBK - 1) / TBK;
  p.nchunk = (p.nwin + kTcChunkTiles - 1) / kTcChunkTiles;
  const int64_t qrows = static_cast<int64_t>(p.B) * p.Hq * p.S;
  if (qrows > 0x7fffffffLL) return SEP_ETOOBIG;
  CUtensorMap mq, mdo;
  if (!sep::make_rows_map(&mq, p.q, qrows, D, TBQ) || !sep::make_rows_map(&mdo, p.dout, qrows, D, TBQ))
    return SEP_ECUDA;
  k_sep_bwd_tc_kv<D><<<dim3(p.nwin + p.nwin * p.nchunk, p.Hkv, p.B), kTcThreads, KvSmem<D>::BYTES, st>>>(p, mq, mdo);
  if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  k_sep_bwd_tc_q<D><<<dim3((p.S + TBQ - 1) / TBQ, p.Hq, p.B), kTcThreads, QSmem<D>::BYTES, st>>>(
      p, static_cast<__nv_bfloat16*>(dq));
  return cudaGetLastError() == cudaSuccess ? SEP_OK : SEP_ECUDA;
}

template <int D>
int launch_bwd(const BwdParams& p0, const void* out, void* dq, void* dk, void* dv, void* ws,
               cudaStream_t st) {
  BwdParams p = p0;
  const BwdWs w = bwd_ws(p.B, p.Hq, p.Hkv, p.S, D);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* delta = reinterpret_cast<float*>(base);
  p.delta = delta;
  p.dq_acc = reinterpret_cast<float*>(base + w.delta);
  p.dk_acc = reinterpret_cast<float*>(base + w.delta + w.dq);
  p.dv_acc = reinterpret_cast<float*>(base + w.delta + w.dq + w.dk);
  constexpr bool tc = tc_backward<D>();  // dq is then written directly, in bf16
  if (tc) {
    if (cudaMemsetAsync(p.dk_acc, 0, w.dk + w.dv, st) != cudaSuccess) return SEP_ECUDA;
  } else if (cudaMemsetAsync(p.dq_acc, 0, w.dq + w.dk + w.dv, st) != cudaSuccess) {
    return SEP_ECUDA;
  }
  const int64_t rows = static_cast<int64_t>(p.B) * p.Hq * p.S;
  k_bwd_delta<D><<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(out), p.dout, delta, rows);
  if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  if (tc) {
    const int rc = launch_bwd_tc<D>(p, dq, st);
    if (rc != SEP_OK) return rc;
  } else {
  constexpr int smem = Smem<D>::BYTES;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(k_sep_bwd<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return SEP_ECUDA;
    attr_done[dev] = true;
  }
  dim3 grid(p.nwin + p.nwin * p.nchunk, p.Hkv, p.B);
  k_sep_bwd<D><<<grid, kThreads, smem, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  }
  const float sc = p.scale_log2 / 1.44269504088896340736f;
  struct {
    const float* acc;
    void* dst;
    int64_t n;
    float mul;
  } conv[3] = {{p.dq_acc, dq, rows * D, sc},
               {p.dk_acc, dk, static_cast<int64_t>(p.B) * p.Hkv * p.S * D, sc},
               {p.dv_acc, dv, static_cast<int64_t>(p.B) * p.Hkv * p.S * D, 1.f}};
  for (auto& c : conv) {
    if (tc && c.dst == dq) continue;  // already written
    const int64_t n4 = c.n / 4;
    const int blocks = static_cast<int>(n4 / 256 + 1 < 148 * 16 ? n4 / 256 + 1 : 148 * 16);
    k_bwd_convert<<<blocks, 256, 0, st>>>(c.acc, static_cast<__nv_bfloat16*>(c.dst), n4, c.mul);
    if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  }
  return sep::launch_status();
}

}  // namespace

extern "C" size_t sep_attn_backward_workspace(int B, int Hq, int Hkv, int S, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Hq % Hkv != 0 || (D != 64 && D != 128)) return 0;
  const BwdWs w = bwd_ws(B, Hq, Hkv, S, D);
  return w.delta + w.dq + w.dk + w.dv;
}

extern "C" int sep_attn_backward(const void* q, const void* k, const void* v, const void* out,
                                 const float* lse, const void* dout, int dtype,
                                 const uint8_t* is_sep, const int32_t* prefix, const int32_t* idx,
                                 int B, int Hq, int Hkv, int S, int D, int a, int n, float scale,
                                 void* dq, void* dk, void* dv, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  if (dtype != SEP_BF16) return SEP_EDTYPE;
  if (D != 64 && D != 128) return SEP_EDTYPE;
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Hq % Hkv != 0 || a < 0 || n < 1) return SEP_EINVAL;
  if (B > 65535 || Hkv > 65535 || static_cast<int64_t>(B) * Hq * S * D >= (1LL << 40))
    return SEP_EINVAL;
  if (!q || !k || !v || !out || !lse || !dout || !is_sep || !prefix || !idx || !dq || !dk || !dv ||
      !workspace)
    return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(k) || !sep::aligned16(v) || !sep::aligned16(out) ||
      !sep::aligned16(dout) || !sep::aligned16(dq) || !sep::aligned16(dk) || !sep::aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return SEP_EALIGN;
  if (workspace_bytes < sep_attn_backward_workspace(B, Hq, Hkv, S, D)) return SEP_EINVAL;
  BwdParams p = {};
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.k = static_cast<const __nv_bfloat16*>(k);
  p.v = static_cast<const __nv_bfloat16*>(v);
  p.dout = static_cast<const __nv_bfloat16*>(dout);
  p.lse = lse;
  p.is_sep = is_sep;
  p.prefix = prefix;
  p.idx = idx;
  p.err = sep::device_error_word();
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.a = a;
  p.n = n;
  p.nwin = (S + BC - 1) / BC;
  p.nchunk = (p.nwin + kChunkTiles - 1) / kChunkTiles;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return D == 64 ? launch_bwd<64>(p, out, dq, dk, dv, workspace, st)
                 : launch_bwd<128>(p, out, dq, dk, dv, workspace, st);
}
