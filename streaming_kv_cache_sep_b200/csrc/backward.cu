// Sep-Attention backward (bf16, D in {64, 128}) on tcgen05 tensor cores.
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
// Key-centric work split for dK and dV.  The kept pairs fall into two
// disjoint families:
//   * global keys (j < a or a separator) are kept by every query i >= j;
//     they are taken 128 at a time from the compact list of global keys, and
//     each block visits the query tiles from its first key's on, split into
//     chunks of ctiles tiles aligned to multiples of ctiles (chunk_tiles<D>)
//     (one work item per block, chunk and kv head);
//   * local keys (all others) are kept only by queries i in [j, j + n); they
//     are taken as 128 consecutive positions, and each block visits the query
//     tiles that reach it, with the global keys of the block masked out.
// dQ is query-centric: each CTA owns 128 queries of one head and visits the
// key blocks its tile keeps; it also forms delta_i from its tile of out and
// dout and writes it for the key-centric kernel, which runs after it.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace {

__device__ __forceinline__ void red_add_v2(float* p, float x, float y) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(x), "f"(y) : "memory");
}

struct BwdParams {
  const __nv_bfloat16 *q, *k, *v, *dout;
  const float* lse;    // [B][Hq][S] natural log
  float* delta;        // [B][Hq][S]: written by the query-centric kernel
  const uint8_t* is_sep;
  const int32_t *prefix, *idx;
  float *dk_acc, *dv_acc;  // fp32 dK, dV rows of the compact global-key lists
  int2* items;             // global-key work items (k_bwd_plan)
  int32_t* item_count;     // their number
  int32_t* err;
  int B, Hq, Hkv, S, a, n;
  int nwin;    // window items per (b, kv head) = ceil(S / 128)
  int ctiles;  // query tiles per chunk of a global-key item (chunk_tiles<D>)
  int nchunk;  // chunks per block of global keys = ceil(ceil(S / 128) / ctiles)
  float scale_log2;
};

// ---------------------------------------------------------------------------
// Two software-pipelined tcgen05 kernels on the operand forms of the forward.
//   k_bwd_kv (key-centric, 128 keys in TMEM lanes, K and V resident): in
//     units of 64 queries of one head (each unit's Q and dO rows stream
//     through a ring of kNst shared-memory stages filled by the tensor-copy
//     engine): S^T = K Q^T and dP^T = V dO^T (SS, N = 64) into one of two
//     score buffers; the compute warps turn them into P^T and dS^T, written
//     back as bf16 over the first 16 columns of each warp's 32; then
//     dV += P^T dO and dK += dS^T Q (TS, B MN-major).  The MMA warp issues
//     the scores of unit u before the gradient products of unit u-1, so the
//     tensor pipe computes while the compute warps work on the other
//     buffer.  TMEM: S0 [0,64) dP0 [64,128) S1 [128,192) dP1 [192,256)
//     dV [256,256+D) dK [256+D,256+2D), and at D = 64 a second dV, dK pair
//     [384,512) for every other item.
//   k_bwd_q (query-centric, 128 queries in TMEM lanes, Q, dO and out
//     resident; delta of each row from dO and out first):
//     over the kept key blocks of its tile as the forward does -- the global
//     keys before the window from the compact list, then the window blocks
//     with the element mask -- in units of 64 keys streamed through the
//     ring: S = Q K^T and dP = dO V^T (SS), dS written back as bf16,
//     dQ += dS K (TS, B = K MN-major).  The CTA owns its queries, so dQ is
//     stored once, as bf16.  TMEM: S0 dP0 S1 dP1 as above, dQ of every
//     other item in [256, 256+D) and [256+D, 256+2D).
// Warps 0-7 are the compute warps (warp w: TMEM lanes 32 (w & 3) .. +31,
// columns [32 (w >> 2), +32) of each 64-column score tile), warp 8
// allocates TMEM and its lane 0 issues the MMAs, warp 9 issues the tensor
// copies and stages the per-unit statistics (key-centric) or global-flag
// words (query-centric).  A ring stage is released by the commit of the
// last product that reads it.  Every wait is bounded.
//
// Key rows: the global keys (initial tokens and separators) are read from a
// compact copy [B, Hkv, S, D] (k_bwd_prep), so every K/V block is one
// tensor copy.  Window keys' dK and dV are owned by one item and stored as
// bf16; the global keys' partial sums go to fp32 rows of the compact list
// (zeroed by k_bwd_prep) and k_bwd_scatter writes them to their positions.

constexpr int TBK = 128;  // keys per block
constexpr int TBQ = 128;  // queries per tile
constexpr int kTcThreads = 320;
constexpr int kNst = 4;           // stages of the 64-row operand ring
constexpr int kT64 = 64 * 128;    // one 64-row x 64-column swizzled tile
constexpr uint32_t kColAcc = 256;    // accumulators: dV, dK (key-centric) / dQ (query-centric)
constexpr int kT128 = 128 * 128;  // one 128-row x 64-column swizzled tile
// Query tiles per chunk of a global-key item, measured per head dimension
// (Llama-3 8k shape at D = 128: 4 tiles 0.541 ms, 8 0.595, 16 0.646;
// Pythia-160M shape at D = 64: 4 tiles 0.239 ms, 8 0.218, 16 0.238).  At
// D = 64 the key-centric kernel double-buffers K and V, so fewer, longer
// items cost no reload bubble.
template <int D>
constexpr int chunk_tiles() { return D == 64 ? 8 : 4; }

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
// TMEM column of the bf16 operand of k-step kk (16 rows of K) of a unit
// whose values were stored by the compute warps at [base + 32 ch, +16)
__device__ __forceinline__ uint32_t unit_acol(uint32_t base, int kk) {
  return base + 32u * static_cast<uint32_t>(kk >> 1) + 8u * static_cast<uint32_t>(kk & 1);
}
// 128 rows starting at `row` of a [rows, D] tensor map into NB 64-column
// swizzled tiles at `dst`, completing on `bar`
template <int D>
__device__ __forceinline__ void load_tile128(uint8_t* dst, const CUtensorMap* map, int32_t row,
                                             uint64_t* bar) {
#pragma unroll
  for (int c = 0; c < D / 64; ++c) sep::tma_load_2d(dst + c * kT128, map, 64 * c, row, bar);
}

// The compact list of global keys of (b, kv head): initial tokens [0,
// min(a, S)), then separators at positions >= a, in order.
struct GlobalList {
  const int32_t* pre;
  const int32_t* ix;
  int a0, total;
  __device__ GlobalList(const BwdParams& p, int b) {
    pre = p.prefix + static_cast<int64_t>(b) * (p.S + 1);
    ix = p.idx + static_cast<int64_t>(b) * p.S;
    a0 = p.a < p.S ? p.a : p.S;
    total = a0 + (pre[p.S] - pre[a0]);
  }
  __device__ int pos(int t) const { return t < a0 ? t : ix[pre[a0] + t - a0]; }
};

// Programmatic launch: let the next grid on the stream start launching
// (pdl_trigger), and wait until the grids before this one have completed
// with their stores visible (pdl_wait; returns at once without a
// programmatic dependency).
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Copies the global keys' K/V rows into the compact buffers (rows past the
// list and up to the next multiple of 128, at least 128 and at most S, are
// zero-filled so whole tiles read finite values) and zeroes the fp32
// dK/dV rows of the list.  One CTA per 64 rows of (b, kv head).
//
// Runs alongside k_bwd_plan (launched just before it, programmatically):
// both read only the index.  CTA (0, 0, 0) waits for the plan grid before
// it ends, so the completion of this grid, which the next launch waits for,
// also implies the plan's.
template <int D>
__global__ void __launch_bounds__(256) k_bwd_prep(const BwdParams p, __nv_bfloat16* __restrict__ kc,
                                                  __nv_bfloat16* __restrict__ vc) {
  constexpr int CH = D / 8;  // 16-byte chunks per bf16 row
  if (threadIdx.x == 0) pdl_trigger();
  const bool chain = (blockIdx.x | blockIdx.y | blockIdx.z) == 0;
  const int g = blockIdx.y, b = blockIdx.z, r0 = blockIdx.x * 64;
  const GlobalList gl(p, b);
  int lim = (gl.total + TBK - 1) / TBK * TBK;
  if (lim < TBK) lim = TBK;
  if (lim > p.S) lim = p.S;
  if (r0 >= lim) {
    if (chain) pdl_wait();
    return;
  }
  const int64_t base = (static_cast<int64_t>(b) * p.Hkv + g) * p.S;
  for (int e = threadIdx.x; e < 64 * CH; e += 256) {
    const int r = r0 + e / CH, c = e % CH;
    if (r >= lim) break;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (r < gl.total) {
      const int pos = gl.pos(r);
      if (pos >= 0 && pos < p.S) {
        kv = reinterpret_cast<const uint4*>(p.k + (base + pos) * D)[c];
        vv = reinterpret_cast<const uint4*>(p.v + (base + pos) * D)[c];
      } else {
        atomicOr(p.err, sep::ERR_BAD_INDEX);
      }
      const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
      reinterpret_cast<float4*>(p.dk_acc + (base + r) * D)[2 * c] = z;
      reinterpret_cast<float4*>(p.dk_acc + (base + r) * D)[2 * c + 1] = z;
      reinterpret_cast<float4*>(p.dv_acc + (base + r) * D)[2 * c] = z;
      reinterpret_cast<float4*>(p.dv_acc + (base + r) * D)[2 * c + 1] = z;
    }
    reinterpret_cast<uint4*>(kc + (base + r) * D)[c] = kv;
    reinterpret_cast<uint4*>(vc + (base + r) * D)[c] = vv;
  }
  if (chain) pdl_wait();
}

// The global keys' fp32 dK (times scale) and dV sums -> bf16 rows at their
// positions.
template <int D>
__global__ void __launch_bounds__(256) k_bwd_scatter(const BwdParams p, float scale,
                                                     __nv_bfloat16* __restrict__ dk,
                                                     __nv_bfloat16* __restrict__ dv) {
  constexpr int CH = D / 8;
  const int g = blockIdx.y, b = blockIdx.z, r0 = blockIdx.x * 64;
  // every CTA waits for the key-centric kernel (its sums), so this grid
  // completes only after it
  pdl_wait();
  const GlobalList gl(p, b);
  if (r0 >= gl.total) return;
  const int64_t base = (static_cast<int64_t>(b) * p.Hkv + g) * p.S;
  for (int e = threadIdx.x; e < 64 * CH; e += 256) {
    const int r = r0 + e / CH, c = e % CH;
    if (r >= gl.total) break;
    const int pos = gl.pos(r);
    if (pos < 0 || pos >= p.S) continue;  // flagged by k_bwd_prep
    const float4* ks = reinterpret_cast<const float4*>(p.dk_acc + (base + r) * D) + 2 * c;
    const float4* vs = reinterpret_cast<const float4*>(p.dv_acc + (base + r) * D) + 2 * c;
    const float4 k0 = ks[0], k1 = ks[1], v0 = vs[0], v1 = vs[1];
    reinterpret_cast<uint4*>(dk + (base + pos) * D)[c] =
        make_uint4(sep::pack_bf16x2(k0.x * scale, k0.y * scale), sep::pack_bf16x2(k0.z * scale, k0.w * scale),
                   sep::pack_bf16x2(k1.x * scale, k1.y * scale), sep::pack_bf16x2(k1.z * scale, k1.w * scale));
    reinterpret_cast<uint4*>(dv + (base + pos) * D)[c] =
        make_uint4(sep::pack_bf16x2(v0.x, v0.y), sep::pack_bf16x2(v0.z, v0.w),
                   sep::pack_bf16x2(v1.x, v1.y), sep::pack_bf16x2(v1.z, v1.w));
  }
}

// Bounded wait by every lane of a warp on the same phase; true on all lanes
// or on none.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int32_t* err) {
  const bool ok = sep::mbar_wait(bar, parity, abort, err);
  return __all_sync(0xffffffffu, ok);
}
// Adds `bytes` of expected tensor-copy data to the current phase of `bar`
// without an arrival.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(sep::smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
// Bits [a, b) of a 32-bit word, a and b clamped to [0, 32].
__device__ __forceinline__ uint32_t bit_range(int a, int b) {
  a = a < 0 ? 0 : (a > 32 ? 32 : a);
  b = b < 0 ? 0 : (b > 32 ? 32 : b);
  if (b <= a) return 0u;
  const uint32_t hi = b >= 32 ? 0xffffffffu : ((1u << b) - 1u);
  return hi & ~((1u << a) - 1u);
}
// One thread's 32 scores s and dP of a unit -> P = 2^(s scale_log2 + nl)
// and dS = P (dP - dl), each packed to bf16 pairs.  Columns whose bit of
// `keep` is clear (MASK) get a score of -inf, so P = 0 and dS = 0 there.
// COLSTATS: nl and dl per column (float4 reads of nl[], dl[]), else the
// row's nl2, dl2.
template <bool MASK, bool COLSTATS>
__device__ __forceinline__ void probs_grads(const uint32_t (&sv)[32], const uint32_t (&dpv)[32],
                                            const float* nl, const float* dl, float2 nl2, float2 dl2,
                                            float2 sc2, uint32_t keep, uint32_t (&pp)[16],
                                            uint32_t (&dd)[16]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    float4 n4 = make_float4(0.f, 0.f, 0.f, 0.f), d4 = n4;
    if constexpr (COLSTATS) {
      n4 = *reinterpret_cast<const float4*>(nl + e);
      d4 = *reinterpret_cast<const float4*>(dl + e);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = e + 2 * h;
      const float2 nn = COLSTATS ? (h ? make_float2(n4.z, n4.w) : make_float2(n4.x, n4.y)) : nl2;
      const float2 dm = COLSTATS ? (h ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y)) : dl2;
      float2 x = sep::ffma2(make_float2(__uint_as_float(sv[f]), __uint_as_float(sv[f + 1])), sc2, nn);
      if constexpr (MASK) {
        x.x = (keep >> f) & 1u ? x.x : -INFINITY;
        x.y = (keep >> (f + 1)) & 1u ? x.y : -INFINITY;
      }
      const float p0 = sep::ex2_approx(x.x), p1 = sep::ex2_approx(x.y);
      const float2 ds = fmul2(make_float2(p0, p1),
                              fsub2(make_float2(__uint_as_float(dpv[f]), __uint_as_float(dpv[f + 1])), dm));
      pp[f / 2] = sep::pack_bf16x2(p0, p1);
      dd[f / 2] = sep::pack_bf16x2(ds.x, ds.y);
    }
  }
}

// ---- work items
//
// Key-centric items: listed by k_bwd_plan (global-key blocks on chunks of
// query tiles, and window blocks of 128 positions).  Query-centric items: (b, head, tile of 128 queries),
// tiles with more kept keys (later positions) first.  Both kernels are
// persistent: CTA c takes items c, c + gridDim.x, ... in order, so every
// role of the CTA walks the same sequence without handing items around.

// The key-centric items, per sequence b and kv head g (b-major, then g):
// for each chunk c of p.ctiles query tiles [c ctiles, +ctiles), the
// global-key items (blocks kb of 128 global keys whose
// first key lies before the chunk's end), then the window items (blocks kb
// of 128 positions): the items a CTA runs side by side read the query tiles
// of one kv head, and the heavier come first.  Entry: (b Hkv + g, kb << 16 | c), with
// c = 0xffff for a window item.  One CTA; warp w takes sequences w, w + 32
// ...: their item counts, then (after one thread's prefix over the
// sequences) the items of (b, g) pairs.  p.item_count[1 + b] holds sequence
// b's offset.
constexpr int kPlanWarps = 32;
constexpr int kPlanCache = 512;  // blocks whose first chunk a warp keeps in shared memory
constexpr int kWindowItem = 0xffff;
__global__ void __launch_bounds__(32 * kPlanWarps) k_bwd_plan(const BwdParams p) {
  if (threadIdx.x == 0) pdl_trigger();  // k_bwd_prep runs alongside
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nT = (p.S + TBQ - 1) / TBQ;
  const int nC = (nT + p.ctiles - 1) / p.ctiles;
  int32_t* const off = p.item_count + 1;
  // chunk of the first tile of block kb of sequence b
  auto first_chunk = [&](const GlobalList& gl, int kb) {
    const int pos = gl.pos(kb * TBK);
    return (pos >= 0 && pos < p.S ? pos : 0) / TBQ / p.ctiles;
  };
  for (int b = warp; b < p.B; b += kPlanWarps) {
    const GlobalList gl(p, b);
    const int nb = (gl.total + TBK - 1) / TBK;
    int n = 0;  // block kb has items for chunks first_chunk .. nC - 1
    for (int kb = lane; kb < nb; kb += 32) n += nC - first_chunk(gl, kb);
#pragma unroll
    for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
    if (lane == 0) off[b] = n + p.nwin;  // items per kv head
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int e = 0;
    for (int b = 0; b < p.B; ++b) {
      const int n = off[b];
      off[b] = e;
      e += n * p.Hkv;
    }
    *p.item_count = e;
  }
  __syncthreads();
  // (b, g) pairs across the warps; each warp caches its blocks' first chunks
  __shared__ int16_t fc_s[kPlanWarps][kPlanCache];
  for (int pr = warp; pr < p.B * p.Hkv; pr += kPlanWarps) {
    const int b = pr / p.Hkv, g = pr % p.Hkv;
    const GlobalList gl(p, b);
    const int nb = (gl.total + TBK - 1) / TBK;
    const bool cached = nb <= kPlanCache;
    if (cached)
      for (int kb = lane; kb < nb; kb += 32) fc_s[warp][kb] = static_cast<int16_t>(first_chunk(gl, kb));
    __syncwarp();
    const int per = ((b + 1 < p.B ? off[b + 1] : *p.item_count) - off[b]) / p.Hkv;  // items per head
    int e = off[b] + g * per;
    for (int c = 0; c < nC; ++c) {
      for (int k0 = 0; k0 < nb; k0 += 32) {
        const int kb = k0 + lane;
        const bool on = kb < nb && (cached ? fc_s[warp][kb] : first_chunk(gl, kb)) <= c;
        const uint32_t m = __ballot_sync(0xffffffffu, on);
        if (on) p.items[e + __popc(m & ((1u << lane) - 1u))] = make_int2(pr, (kb << 16) | c);
        e += __popc(m);
      }
    }
    for (int kb = lane; kb < p.nwin; kb += 32) p.items[e + kb] = make_int2(pr, (kb << 16) | kWindowItem);
    __syncwarp();
  }
}

struct KvItem {
  int b, g, kb, t0, ntile;
  int nh;  // 64-row units per query head: two per tile, less a last half no row of which keeps a key
  bool window;
};
__device__ __forceinline__ KvItem kv_item(const BwdParams& p, int i) {
  KvItem it;
  const int nT = (p.S + TBQ - 1) / TBQ;
  const int2 ent = p.items[i];
  it.b = ent.x / p.Hkv;
  it.g = ent.x % p.Hkv;
  it.kb = ent.y >> 16;
  const int c = ent.y & 0xffff;
  if (c != kWindowItem) {
    const GlobalList gl(p, it.b);
    const int pos = gl.pos(it.kb * TBK);
    const int first = (pos >= 0 && pos < p.S ? pos : 0) / TBQ, c0 = c * p.ctiles;
    it.t0 = first > c0 ? first : c0;
    const int t1 = c0 + p.ctiles < nT ? c0 + p.ctiles : nT;
    it.ntile = t1 - it.t0;
    it.window = false;
  } else {
    it.t0 = it.kb;
    const int last = it.kb * TBK + TBK - 1 + p.n - 1;
    it.ntile = (last < p.S - 1 ? last : p.S - 1) / TBQ + 1 - it.t0;
    it.window = true;
  }
  // the last query that keeps a key of the item: the window's end (window
  // keys), or the sequence's (global keys); at a short window (n <= 64) the
  // second half of a window item's last tile lies past it
  int lastq = it.window ? it.kb * TBK + TBK - 1 + p.n - 1 : p.S - 1;
  if (lastq > p.S - 1) lastq = p.S - 1;
  it.nh = 2 * it.ntile - ((it.t0 + it.ntile - 1) * TBQ + 64 > lastq ? 1 : 0);
  return it;
}
// Unit u of a key-centric item: query head u / nh (of the kv head's group),
// tile t0 + (u % nh) / 2, rows [64 ((u % nh) & 1), +64) of the tile.
__device__ __forceinline__ int kv_unit_head(const KvItem& it, int u) { return u / it.nh; }
__device__ __forceinline__ int kv_unit_tile(const KvItem& it, int u) { return it.t0 + ((u % it.nh) >> 1); }
__device__ __forceinline__ int kv_unit_half(const KvItem& it, int u) { return (u % it.nh) & 1; }

// An item and this compute thread's key row in it: position jp, and
// whether the item's queries keep it (window items leave global keys out).
struct KvRow {
  KvItem it;
  int jp, use;
};
__device__ __forceinline__ KvRow kv_row(const BwdParams& p, int i, int r) {
  KvRow x;
  x.it = kv_item(p, i);
  x.jp = -1;
  x.use = 0;
  if (x.it.window) {
    const int q = x.it.kb * TBK + r;
    if (q < p.S) {
      x.jp = q;
      x.use = !(q < p.a || p.is_sep[static_cast<int64_t>(x.it.b) * p.S + q]);
    }
  } else {
    const GlobalList gl(p, x.it.b);
    const int t = x.it.kb * TBK + r;
    if (t < gl.total) {
      x.jp = gl.pos(t);
      x.use = 1;
    }
  }
  return x;
}

// Shared memory of the key-centric kernel: KVB buffers of an item's K and V
// [128][D] (swizzled 64-column tiles; two buffers where they fit, so the
// next item's keys load during the current one); a ring of kNst unit
// stages, each the unit's Q and dO rows [64][D]; -lse (log2 domain) and
// delta [kNst][64] fp32.
template <int D>
struct KvSmem {
  static constexpr int NB = D / 64;
  static constexpr int KVB = D == 64 ? 2 : 1;
  static constexpr int KVSZ = 2 * NB * kT128;  // K tiles, then V tiles
  static constexpr int RING = KVB * KVSZ;
  static constexpr int STAGE = 2 * NB * kT64;  // Q tiles, then dO tiles
  static constexpr int LSE = RING + kNst * STAGE;
  static constexpr int DEL = LSE + kNst * 64 * 4;
  static constexpr int BYTES = DEL + kNst * 64 * 4 + 1024;  // + alignment slack
};
struct KvBars {
  uint64_t kv_full[2], kv_free[2], st_full[kNst], st_free[kNst], s_full[2], p_full[2];
  uint64_t fin[2], acc_free[2], drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_bwd_kv(const BwdParams p, const __grid_constant__ CUtensorMap map_q,
             const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_k,
             const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kc,
             const __grid_constant__ CUtensorMap map_vc, __nv_bfloat16* __restrict__ dk,
             __nv_bfloat16* __restrict__ dv) {
  using Sm = KvSmem<D>;
  constexpr int NB = D / 64;
  constexpr int KVB = Sm::KVB;
  // dV, dK accumulator buffers (columns [256, 512)): two where they fit, so
  // an item's products need not wait for the previous item's read-out
  constexpr int ACCB = D == 64 ? 2 : 1;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* const smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ KvBars bars;
  const uint32_t sb_ = sep::smem_u32(smem);
  float* const lse_s = reinterpret_cast<float*>(smem + Sm::LSE);
  float* const del_s = reinterpret_cast<float*>(smem + Sm::DEL);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, G = p.Hq / p.Hkv;
  // first row of unit u of item `it` in the [B * Hq * S] view
  auto unit_row = [&](const KvItem& it, int u) -> int64_t {
    return (static_cast<int64_t>(it.b) * p.Hq + it.g * G + kv_unit_head(it, u)) * S +
           kv_unit_tile(it, u) * TBQ + 64 * kv_unit_half(it, u);
  };

  if (threadIdx.x == 9 * 32) {
    for (int i = 0; i < KVB; ++i) {
      sep::mbar_init(&bars.kv_full[i], 1);
      sep::mbar_init(&bars.kv_free[i], 1);
    }
    for (int i = 0; i < kNst; ++i) {
      sep::mbar_init(&bars.st_full[i], 32);  // the load warp's lanes, after the statistics
      sep::mbar_init(&bars.st_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      sep::mbar_init(&bars.s_full[i], 1);
      sep::mbar_init(&bars.p_full[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      sep::mbar_init(&bars.fin[i], 1);
      sep::mbar_init(&bars.acc_free[i], 8);
    }
    sep::mbar_init(&bars.drain, 1);
    sep::mbar_fence_init();
    pdl_trigger();  // the next kernel's CTAs take SMs as this grid's retire
  }
  if (warp == 8) {
    sep::tmem_alloc(&bars.tmem_base, 512);
    sep::tmem_relinquish();
  }
  // everything above overlaps the previous kernel; its outputs are read below
  pdl_wait();
  if (threadIdx.x == 9 * 32)  // a wait of an earlier CTA gave up: this one ends at its first wait too
    bars.abort = (*reinterpret_cast<volatile int32_t*>(p.err) & sep::ERR_WAIT_TIMEOUT) ? 1 : 0;
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  const int nitems = *p.item_count;  // written by k_bwd_plan
  const uint32_t tmem = bars.tmem_base;
  volatile int* abort = &bars.abort;

  if (warp < 8) {
    // ------------------------------------------------ compute warps
    const int lq = warp & 3, ch = warp >> 2;
    const int r = 32 * lq + lane;  // key row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * lq) << 16;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const float sc = p.scale_log2 * 0.69314718055994530942f;
    bool ok = true;
    uint32_t U = 0, I = 0;  // units and items of this CTA so far
    // every role decodes the next item (dependent global loads) while it
    // works on the current one
    KvRow cur = blockIdx.x < nitems ? kv_row(p, blockIdx.x, r) : KvRow{};
    for (int i = blockIdx.x; i < nitems && ok; i += gridDim.x, ++I) {
      const KvRow nxt = i + static_cast<int>(gridDim.x) < nitems ? kv_row(p, i + gridDim.x, r) : cur;
      const KvItem it = cur.it;
      const int jp = cur.jp, use = cur.use;
      cur = nxt;
      const int nunit = G * it.nh;
      const int64_t kvrow0 = (static_cast<int64_t>(it.b) * p.Hkv + it.g) * S;
      for (int u = 0; u < nunit; ++u) {
        const uint32_t gu = U + u;
        const int hh = kv_unit_half(it, u), sb = gu & 1, st = gu % kNst;
        const int i0 = kv_unit_tile(it, u) * TBQ;
        if (!warp_wait(&bars.st_full[st], (gu / kNst) & 1, abort, p.err) ||
            !warp_wait(&bars.s_full[sb], (gu >> 1) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        sep::tc_fence_after();
        // the unit columns this key row keeps: [qa, qb) relative to column
        // 64 hh + 32 ch of the tile
        int qa = 0, qb = 0;
        if (use && jp >= 0) {
          qa = jp - i0 > 0 ? jp - i0 : 0;
          qb = S - i0 < TBQ ? S - i0 : TBQ;
          if (it.window && jp + p.n - i0 < qb) qb = jp + p.n - i0;
        }
        const int c0 = 64 * hh + 32 * ch;
        const uint32_t keep = bit_range(qa - c0, qb - c0);
        const uint32_t cs = 128u * sb + 32u * ch;
        uint32_t pp[16], dd[16];
        if (__all_sync(0xffffffffu, keep == 0u)) {
          // no column of the warp's rows is kept: P^T and dS^T are zero
#pragma unroll
          for (int e = 0; e < 16; ++e) pp[e] = dd[e] = 0u;
        } else {
          uint32_t sv[32], dv_[32];
          sep::tmem_ld32(tmem + lane_base + cs, sv);
          sep::tmem_ld32(tmem + lane_base + cs + 64, dv_);
          sep::tmem_wait_ld_r32(sv);
          sep::tmem_wait_ld_r32(dv_);
          const float* nl = lse_s + st * 64 + 32 * ch;
          const float* dl = del_s + st * 64 + 32 * ch;
          const float2 z2 = make_float2(0.f, 0.f);
          if (__all_sync(0xffffffffu, keep == 0xffffffffu))
            probs_grads<false, true>(sv, dv_, nl, dl, z2, z2, sc2, keep, pp, dd);
          else
            probs_grads<true, true>(sv, dv_, nl, dl, z2, z2, sc2, keep, pp, dd);
        }
        sep::tmem_st16(tmem + lane_base + cs, pp);
        sep::tmem_st16(tmem + lane_base + cs + 64, dd);
        sep::tmem_wait_st();
        sep::tc_fence_before();
        __syncwarp();
        if (lane == 0) sep::mbar_arrive(&bars.p_full[sb]);
      }
      const int abuf = I % ACCB;
      if (!ok || !warp_wait(&bars.fin[abuf], (I / ACCB) & 1, abort, p.err)) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
      // dK and dV of this key row, columns [D/2 ch, +D/2): every lane loads
      // (warp-wide); once the last load is in, the accumulators are handed
      // back for a later item.  A window key is stored as bf16, a global
      // key's partial sum is added to its fp32 row of the compact list.
      const bool mine = jp >= 0 && use;
      const int64_t row = kvrow0 + (it.window ? (mine ? jp : 0) : it.kb * TBK + r);
      const uint32_t cdv = kColAcc + 2u * D * abuf, cdk = cdv + D;
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t kv[32], vv[32];
        const int col = (D / 2) * ch + 32 * c;
        sep::tmem_ld32(tmem + lane_base + cdk + col, kv);
        sep::tmem_ld32(tmem + lane_base + cdv + col, vv);
        sep::tmem_wait_ld_r32(kv);
        sep::tmem_wait_ld_r32(vv);
        if (c == D / 64 - 1) {
          sep::tc_fence_before();
          __syncwarp();
          if (lane == 0) sep::mbar_arrive(&bars.acc_free[abuf]);
        }
        if (!mine) continue;
        if (it.window) {
          uint4* kd = reinterpret_cast<uint4*>(dk + row * D + col);
          uint4* vd = reinterpret_cast<uint4*>(dv + row * D + col);
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4) {
            kd[u4] = make_uint4(sep::pack_bf16x2(__uint_as_float(kv[8 * u4]) * sc, __uint_as_float(kv[8 * u4 + 1]) * sc),
                                sep::pack_bf16x2(__uint_as_float(kv[8 * u4 + 2]) * sc, __uint_as_float(kv[8 * u4 + 3]) * sc),
                                sep::pack_bf16x2(__uint_as_float(kv[8 * u4 + 4]) * sc, __uint_as_float(kv[8 * u4 + 5]) * sc),
                                sep::pack_bf16x2(__uint_as_float(kv[8 * u4 + 6]) * sc, __uint_as_float(kv[8 * u4 + 7]) * sc));
            vd[u4] = make_uint4(sep::pack_bf16x2(__uint_as_float(vv[8 * u4]), __uint_as_float(vv[8 * u4 + 1])),
                                sep::pack_bf16x2(__uint_as_float(vv[8 * u4 + 2]), __uint_as_float(vv[8 * u4 + 3])),
                                sep::pack_bf16x2(__uint_as_float(vv[8 * u4 + 4]), __uint_as_float(vv[8 * u4 + 5])),
                                sep::pack_bf16x2(__uint_as_float(vv[8 * u4 + 6]), __uint_as_float(vv[8 * u4 + 7])));
          }
        } else {
          float* kp = p.dk_acc + row * D + col;
          float* vp = p.dv_acc + row * D + col;
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            red_add_v2(kp + e, __uint_as_float(kv[e]), __uint_as_float(kv[e + 1]));
            red_add_v2(vp + e, __uint_as_float(vv[e]), __uint_as_float(vv[e + 1]));
          }
        }
      }
      U += nunit;
    }
  } else if (warp == 8) {
    if (lane == 0) {
      // ---------------------------------------------- MMA issue (one thread)
      constexpr uint32_t id_s = idesc_mn(128, 64, false, false);
      constexpr uint32_t id_o = idesc_mn(128, D, false, true);
      bool ok = true;
      uint32_t U = 0, I = 0;
      KvItem cur = blockIdx.x < nitems ? kv_item(p, blockIdx.x) : KvItem{};
      for (int i = blockIdx.x; i < nitems && ok; i += gridDim.x, ++I) {
        const KvItem it = cur;
        cur = i + static_cast<int>(gridDim.x) < nitems ? kv_item(p, i + gridDim.x) : cur;
        const int nunit = G * it.nh;
        const int kbuf = I % KVB, abuf = I % ACCB;
        const uint32_t cdv = kColAcc + 2u * D * abuf, cdk = cdv + D;
        if (!sep::mbar_wait(&bars.kv_full[kbuf], (I / KVB) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        const uint64_t dK = sep::smem_desc_sw128(sb_ + kbuf * Sm::KVSZ, 16);
        const uint64_t dV = sep::smem_desc_sw128(sb_ + kbuf * Sm::KVSZ + NB * kT128, 16);
        for (int u = 0; u <= nunit; ++u) {
          if (u < nunit) {
            // scores of unit u into buffer (U + u) & 1 (its previous
            // contents were read by the products issued before this point)
            const uint32_t gu = U + u;
            const int st = gu % kNst;
            if (!sep::mbar_wait(&bars.st_full[st], (gu / kNst) & 1, abort, p.err)) {
              ok = false;
              break;
            }
            sep::tc_fence_after();
            const uint32_t qa = sb_ + Sm::RING + st * Sm::STAGE, oa = qa + NB * kT64;
            const uint64_t dQ = sep::smem_desc_sw128(qa, 16), dO = sep::smem_desc_sw128(oa, 16);
            const uint32_t cs = 128u * (gu & 1);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t kofs = static_cast<uint64_t>(((kk / 4) * kT128 + (kk % 4) * 32) >> 4);
              const uint64_t qofs = static_cast<uint64_t>(((kk / 4) * kT64 + (kk % 4) * 32) >> 4);
              sep::mma_bf16_ss(tmem + cs, dK + kofs, dQ + qofs, id_s, kk > 0 ? 1u : 0u);
              sep::mma_bf16_ss(tmem + cs + 64, dV + kofs, dO + qofs, id_s, kk > 0 ? 1u : 0u);
            }
            sep::mma_commit(&bars.s_full[gu & 1]);
            if (u == nunit - 1) sep::mma_commit(&bars.kv_free[kbuf]);  // the item's K, V are read
          }
          if (u >= 1) {
            // gradient products of unit u - 1 once its P^T and dS^T are in
            // (and, for the item's first, once the previous item's dK, dV
            // have been read out)
            const uint32_t w = U + u - 1;
            const int wst = w % kNst;
            if (!sep::mbar_wait(&bars.p_full[w & 1], (w >> 1) & 1, abort, p.err) ||
                (u == 1 && I >= ACCB &&
                 !sep::mbar_wait(&bars.acc_free[abuf], ((I - ACCB) / ACCB) & 1, abort, p.err))) {
              ok = false;
              break;
            }
            sep::tc_fence_after();
            const uint32_t qa = sb_ + Sm::RING + wst * Sm::STAGE, oa = qa + NB * kT64;
            const uint64_t dQmn = sep::smem_desc_sw128(qa, kT64), dOmn = sep::smem_desc_sw128(oa, kT64);
            const uint32_t cs = 128u * (w & 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = static_cast<uint64_t>(kk * (2048 >> 4));
              const uint32_t acc = (u > 1 || kk > 0) ? 1u : 0u;
              sep::mma_bf16_ts(tmem + cdv, tmem + unit_acol(cs, kk), dOmn + off, id_o, acc);
              sep::mma_bf16_ts(tmem + cdk, tmem + unit_acol(cs + 64, kk), dQmn + off, id_o, acc);
            }
            sep::mma_commit(&bars.st_free[wst]);  // the stage may be refilled
          }
        }
        if (!ok) break;
        sep::mma_commit(&bars.fin[abuf]);
        U += nunit;
      }
      sep::mma_commit(&bars.drain);  // every MMA completes before TMEM is released
      int keep = 0;
      sep::mbar_wait(&bars.drain, 0, &keep, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ loads (warp 9)
    // Per item: its K and V once their buffer is free; per unit: the copies
    // once its stage is free, the unit's -lse (log2 domain) and delta (rows
    // lane, lane + 32), then the 32 arrivals that complete the stage with
    // its bytes.
    uint32_t U = 0, I = 0;
    uint32_t issued_u = 0, issued_i = 0;  // copies started (units, items)
    bool ok = true;
    KvItem cur = blockIdx.x < nitems ? kv_item(p, blockIdx.x) : KvItem{};
    for (int i = blockIdx.x; i < nitems && ok; i += gridDim.x, ++I) {
      const KvItem it = cur;
      cur = i + static_cast<int>(gridDim.x) < nitems ? kv_item(p, i + gridDim.x) : cur;
      const int nunit = G * it.nh;
      const int kbuf = I % KVB;
      bool go = true;
      if (lane == 0) {
        if (I >= KVB) go = sep::mbar_wait(&bars.kv_free[kbuf], ((I - KVB) / KVB) & 1, abort, p.err);
        if (go) {
          sep::mbar_arrive_expect_tx(&bars.kv_full[kbuf], Sm::KVSZ);
          const int32_t row = static_cast<int32_t>((static_cast<int64_t>(it.b) * p.Hkv + it.g) * S + it.kb * TBK);
          load_tile128<D>(smem + kbuf * Sm::KVSZ, it.window ? &map_k : &map_kc, row, &bars.kv_full[kbuf]);
          load_tile128<D>(smem + kbuf * Sm::KVSZ + NB * kT128, it.window ? &map_v : &map_vc, row,
                          &bars.kv_full[kbuf]);
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      issued_i = I + 1;
      for (int u = 0; u < nunit; ++u) {
        const uint32_t gu = U + u;
        const int st = gu % kNst;
        const int64_t row0 = unit_row(it, u);
        const int i0 = kv_unit_tile(it, u) * TBQ + 64 * kv_unit_half(it, u);
        float nlr[2], dlr[2];  // loads in flight during the wait below
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int e = lane + 32 * m;
          nlr[m] = i0 + e < S ? -p.lse[row0 + e] * 1.44269504088896340736f : 0.f;
          dlr[m] = i0 + e < S ? p.delta[row0 + e] : 0.f;
        }
        if (lane == 0) {
          if (gu >= kNst) go = sep::mbar_wait(&bars.st_free[st], ((gu / kNst) - 1) & 1, abort, p.err);
          if (go) {
            uint8_t* dst = smem + Sm::RING + st * Sm::STAGE;
            mbar_expect_tx(&bars.st_full[st], Sm::STAGE);
#pragma unroll
            for (int c = 0; c < NB; ++c) {
              sep::tma_load_2d(dst + c * kT64, &map_q, 64 * c, static_cast<int32_t>(row0), &bars.st_full[st]);
              sep::tma_load_2d(dst + (NB + c) * kT64, &map_do, 64 * c, static_cast<int32_t>(row0), &bars.st_full[st]);
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        issued_u = gu + 1;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          lse_s[st * 64 + lane + 32 * m] = nlr[m];
          del_s[st * 64 + lane + 32 * m] = dlr[m];
        }
        sep::mbar_arrive(&bars.st_full[st]);
      }
      U += nunit;
    }
    // after an abort, let the started copies land before the CTA can exit
    if (lane == 0 && *abort) {
      int dummy = 0;
      for (uint32_t j = issued_i > KVB ? issued_i - KVB : 0; j < issued_i; ++j)
        sep::mbar_wait(&bars.kv_full[j % KVB], (j / KVB) & 1, &dummy, nullptr);
      for (uint32_t g2 = issued_u > kNst ? issued_u - kNst : 0; g2 < issued_u; ++g2)
        sep::mbar_wait(&bars.st_full[g2 % kNst], (g2 / kNst) & 1, &dummy, nullptr);
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

// Shared memory of the query-centric kernel: QB buffers of an item's Q, dO
// and out [128][D] (swizzled 64-column tiles; two where they fit); a ring of kNst
// unit stages, each the unit's K and V rows [64][D]; the global flags of
// each stage's keys as [kNst][2] 32-bit words (bit k of word m: key 32 m + k
// of the unit).
template <int D>
struct QSmem {
  static constexpr int NB = D / 64;
  static constexpr int QB = D == 64 ? 2 : 1;
  static constexpr int QSZ = 3 * NB * kT128;  // Q tiles, dO tiles, out tiles
  static constexpr int RING = QB * QSZ;
  static constexpr int STAGE = 2 * NB * kT64;  // K tiles, then V tiles
  static constexpr int GLB = RING + kNst * STAGE;
  static constexpr int BYTES = GLB + 1024 + 1024;
};
struct QBars {
  uint64_t q_full[2], q_free[2], st_full[kNst], st_free[kNst], s_full[2], p_full[2];
  uint64_t fin[2], acc_free[2], drain;
  uint32_t tmem_base;
  int abort;
};
struct QItem {
  int b, h, t, lo, qlast, nglo, nbg, nblk;
  int nunit;  // 64-key units: two per block, less a last window half past the tile's last row
};
__device__ __forceinline__ QItem q_item(const BwdParams& p, int i) {
  QItem it;
  const int nT = (p.S + TBQ - 1) / TBQ;
  const int bh = p.B * p.Hq;
  it.t = nT - 1 - i / bh;
  it.h = (i % bh) % p.Hq;
  it.b = (i % bh) / p.Hq;
  const int i0 = it.t * TBQ;
  it.qlast = (i0 + TBQ < p.S ? i0 + TBQ : p.S) - 1;
  // the tile's kept keys: global keys before the first row's window (the
  // head of the compact list), then the window positions [lo, qlast]
  it.lo = i0 - p.n + 1 > 0 ? i0 - p.n + 1 : 0;
  const int32_t* pre = p.prefix + static_cast<int64_t>(it.b) * (p.S + 1);
  const int al = p.a < it.lo ? p.a : it.lo;
  it.nglo = al + (pre[it.lo] - pre[al]);
  it.nbg = (it.nglo + TBK - 1) / TBK;
  it.nblk = it.nbg + (it.qlast - it.lo + TBK) / TBK;
  // the last window block's second half starts past qlast at a short
  // window (n <= 64): no row of the tile keeps any of its keys
  it.nunit = 2 * it.nblk - (it.lo + (it.nblk - it.nbg - 1) * TBK + 64 > it.qlast ? 1 : 0);
  return it;
}

template <int D>
__global__ void __launch_bounds__(kTcThreads, 1)
    k_bwd_q(const BwdParams p, const __grid_constant__ CUtensorMap map_q,
            const __grid_constant__ CUtensorMap map_do, const __grid_constant__ CUtensorMap map_o,
            const __grid_constant__ CUtensorMap map_k,
            const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kc,
            const __grid_constant__ CUtensorMap map_vc, __nv_bfloat16* __restrict__ dq) {
  using Sm = QSmem<D>;
  constexpr int NB = D / 64;
  constexpr int QB = Sm::QB;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* const smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ QBars bars;
  const uint32_t sb_ = sep::smem_u32(smem);
  uint32_t* const glb_w = reinterpret_cast<uint32_t*>(smem + Sm::GLB);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = p.S, G = p.Hq / p.Hkv;
  const int nitems = p.B * p.Hq * ((S + TBQ - 1) / TBQ);
  // unit u of item `it`: keys [64 (u & 1), +64) of block u >> 1 -- rows of
  // the compact list (global blocks) or positions (window blocks)
  auto unit_key = [&](const QItem& it, int u) -> int {
    const int j = u >> 1;
    return (j < it.nbg ? j * TBK : it.lo + (j - it.nbg) * TBK) + 64 * (u & 1);
  };

  if (threadIdx.x == 9 * 32) {
    for (int i = 0; i < QB; ++i) {
      sep::mbar_init(&bars.q_full[i], 1);
      sep::mbar_init(&bars.q_free[i], 9);  // the last score products' commit, the 8 compute warps
    }
    for (int i = 0; i < kNst; ++i) {
      sep::mbar_init(&bars.st_full[i], 32);
      sep::mbar_init(&bars.st_free[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      sep::mbar_init(&bars.s_full[i], 1);
      sep::mbar_init(&bars.p_full[i], 8);
    }
    for (int i = 0; i < 2; ++i) {
      sep::mbar_init(&bars.fin[i], 1);
      sep::mbar_init(&bars.acc_free[i], 8);
    }
    sep::mbar_init(&bars.drain, 1);
    sep::mbar_fence_init();
    pdl_trigger();  // the next kernel's CTAs take SMs as this grid's retire
  }
  if (warp == 8) {
    sep::tmem_alloc(&bars.tmem_base, 512);
    sep::tmem_relinquish();
  }
  // everything above overlaps the previous kernel; its outputs are read below
  pdl_wait();
  if (threadIdx.x == 9 * 32)  // a wait of an earlier CTA gave up: this one ends at its first wait too
    bars.abort = (*reinterpret_cast<volatile int32_t*>(p.err) & sep::ERR_WAIT_TIMEOUT) ? 1 : 0;
  sep::tc_fence_before();
  __syncthreads();
  sep::tc_fence_after();
  const uint32_t tmem = bars.tmem_base;
  volatile int* abort = &bars.abort;

  if (warp < 8) {
    const int lq = warp & 3, ch = warp >> 2;
    const int r = 32 * lq + lane;  // query row = TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(32 * lq) << 16;
    const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
    const float sc = p.scale_log2 * 0.69314718055994530942f;
    bool ok = true;
    uint32_t U = 0, I = 0;
    // every role decodes the next item while it works on the current one
    auto row_nl = [&](const QItem& x) {
      const int i = x.t * TBQ + r;
      return i < S ? -p.lse[(static_cast<int64_t>(x.b) * p.Hq + x.h) * S + i] * 1.44269504088896340736f : 0.f;
    };
    QItem cur = blockIdx.x < nitems ? q_item(p, blockIdx.x) : QItem{};
    float cur_nl = blockIdx.x < nitems ? row_nl(cur) : 0.f;
    for (int ii = blockIdx.x; ii < nitems && ok; ii += gridDim.x, ++I) {
      const QItem it = cur;
      const float nlse2 = cur_nl;
      if (ii + static_cast<int>(gridDim.x) < nitems) {
        cur = q_item(p, ii + gridDim.x);
        cur_nl = row_nl(cur);
      }
      const int nunit = it.nunit;
      const int i = it.t * TBQ + r;
      const int64_t qrow0 = (static_cast<int64_t>(it.b) * p.Hq + it.h) * S;
      // delta of this row: dout . out over its D columns (both warps of the
      // lane quarter form it; the first stores it for the key-centric kernel)
      const int qbuf = I % QB;
      if (!warp_wait(&bars.q_full[qbuf], (I / QB) & 1, abort, p.err)) {
        ok = false;
        break;
      }
      float dl = 0.f;
      {
        const uint8_t* dos = smem + qbuf * Sm::QSZ + NB * kT128;
        const uint8_t* os = dos + NB * kT128;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint32_t off = static_cast<uint32_t>((c >> 3) * kT128 + r * 128 + ((((c & 7) ^ (r & 7))) << 4));
          const uint4 a4 = *reinterpret_cast<const uint4*>(dos + off);
          const uint4 b4 = *reinterpret_cast<const uint4*>(os + off);
          const uint32_t aw[4] = {a4.x, a4.y, a4.z, a4.w}, bw[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            dl = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), dl);
            dl = fmaf(__uint_as_float(aw[e] & 0xffff0000u), __uint_as_float(bw[e] & 0xffff0000u), dl);
          }
        }
      }
      __syncwarp();
      if (lane == 0) sep::mbar_arrive(&bars.q_free[qbuf]);  // this warp is done with dO and out
      if (i >= S) dl = 0.f;
      else if (ch == 0) p.delta[qrow0 + i] = dl;
      const float2 nl2 = make_float2(nlse2, nlse2), dl2 = make_float2(dl, dl);
      for (int u = 0; u < nunit; ++u) {
        const uint32_t gu = U + u;
        const int j = u >> 1, hh = u & 1, sb = gu & 1, st = gu % kNst;
        if (!warp_wait(&bars.st_full[st], (gu / kNst) & 1, abort, p.err) ||
            !warp_wait(&bars.s_full[sb], (gu >> 1) & 1, abort, p.err)) {
          ok = false;  // (st_full: the unit's global-flag words are in shared memory)
          break;
        }
        sep::tc_fence_after();
        // the unit's key columns this query row keeps, relative to column
        // c0 = 64 hh + 32 ch of the block: global blocks, every listed key;
        // window blocks (contiguous positions from `base`), keys at or
        // before the row (and the tile), within n - 1 of it unless global
        const int c0 = 64 * hh + 32 * ch;
        uint32_t keep;
        if (j < it.nbg) {
          keep = bit_range(-c0, (it.nglo - j * TBK < TBK ? it.nglo - j * TBK : TBK) - c0);
        } else {
          const int base = it.lo + (j - it.nbg) * TBK;
          int kb2 = i - base + 1;  // keys at positions <= i, in the tile's range
          if (kb2 > it.qlast - base + 1) kb2 = it.qlast - base + 1;
          keep = bit_range(-c0, kb2 - c0) &
               (bit_range(i - base - p.n + 1 - c0, 32) | glb_w[st * 2 + ch]);
        }
        if (i >= S) keep = 0u;
        const uint32_t cs = 128u * sb + 32u * ch;
        uint32_t pp[16], dd[16];
        if (__all_sync(0xffffffffu, keep == 0u)) {
#pragma unroll
          for (int e = 0; e < 16; ++e) dd[e] = 0u;
        } else {
          uint32_t sv[32], dv_[32];
          sep::tmem_ld32(tmem + lane_base + cs, sv);
          sep::tmem_ld32(tmem + lane_base + cs + 64, dv_);
          sep::tmem_wait_ld_r32(sv);
          sep::tmem_wait_ld_r32(dv_);
          if (__all_sync(0xffffffffu, keep == 0xffffffffu))
            probs_grads<false, false>(sv, dv_, nullptr, nullptr, nl2, dl2, sc2, keep, pp, dd);
          else
            probs_grads<true, false>(sv, dv_, nullptr, nullptr, nl2, dl2, sc2, keep, pp, dd);
        }
        sep::tmem_st16(tmem + lane_base + cs, dd);
        sep::tmem_wait_st();
        sep::tc_fence_before();
        __syncwarp();
        if (lane == 0) sep::mbar_arrive(&bars.p_full[sb]);
      }
      const int abuf = I & 1;
      if (!ok || !warp_wait(&bars.fin[abuf], (I >> 1) & 1, abort, p.err)) {
        ok = false;
        break;
      }
      sep::tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 64; ++c) {
        uint32_t qv[32];
        const int col = (D / 2) * ch + 32 * c;
        sep::tmem_ld32(tmem + lane_base + kColAcc + D * abuf + col, qv);
        sep::tmem_wait_ld_r32(qv);
        if (c == D / 64 - 1) {
          sep::tc_fence_before();
          __syncwarp();
          if (lane == 0) sep::mbar_arrive(&bars.acc_free[abuf]);
        }
        if (i < S) {
          uint4* dst = reinterpret_cast<uint4*>(dq + (qrow0 + i) * D + col);
#pragma unroll
          for (int u4 = 0; u4 < 4; ++u4)
            dst[u4] = make_uint4(sep::pack_bf16x2(__uint_as_float(qv[8 * u4]) * sc, __uint_as_float(qv[8 * u4 + 1]) * sc),
                                 sep::pack_bf16x2(__uint_as_float(qv[8 * u4 + 2]) * sc, __uint_as_float(qv[8 * u4 + 3]) * sc),
                                 sep::pack_bf16x2(__uint_as_float(qv[8 * u4 + 4]) * sc, __uint_as_float(qv[8 * u4 + 5]) * sc),
                                 sep::pack_bf16x2(__uint_as_float(qv[8 * u4 + 6]) * sc, __uint_as_float(qv[8 * u4 + 7]) * sc));
        }
      }
      U += nunit;
    }
  } else if (warp == 8) {
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_mn(128, 64, false, false);
      constexpr uint32_t id_o = idesc_mn(128, D, false, true);
      bool ok = true;
      uint32_t U = 0, I = 0;
      QItem cur = blockIdx.x < nitems ? q_item(p, blockIdx.x) : QItem{};
      for (int ii = blockIdx.x; ii < nitems && ok; ii += gridDim.x, ++I) {
        const QItem it = cur;
        cur = ii + static_cast<int>(gridDim.x) < nitems ? q_item(p, ii + gridDim.x) : cur;
        const int nunit = it.nunit;
        const int qbuf = I % QB, abuf = I & 1;
        const uint32_t cdq = kColAcc + static_cast<uint32_t>(D) * abuf;
        if (!sep::mbar_wait(&bars.q_full[qbuf], (I / QB) & 1, abort, p.err)) {
          ok = false;
          break;
        }
        const uint64_t dQ = sep::smem_desc_sw128(sb_ + qbuf * Sm::QSZ, 16);
        const uint64_t dO = sep::smem_desc_sw128(sb_ + qbuf * Sm::QSZ + NB * kT128, 16);
        for (int u = 0; u <= nunit; ++u) {
          if (u < nunit) {
            const uint32_t gu = U + u;
            const int st = gu % kNst;
            if (!sep::mbar_wait(&bars.st_full[st], (gu / kNst) & 1, abort, p.err)) {
              ok = false;
              break;
            }
            sep::tc_fence_after();
            const uint32_t ka = sb_ + Sm::RING + st * Sm::STAGE, va = ka + NB * kT64;
            const uint64_t dK = sep::smem_desc_sw128(ka, 16), dV = sep::smem_desc_sw128(va, 16);
            const uint32_t cs = 128u * (gu & 1);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t oq = static_cast<uint64_t>(((kk / 4) * kT128 + (kk % 4) * 32) >> 4);
              const uint64_t okv = static_cast<uint64_t>(((kk / 4) * kT64 + (kk % 4) * 32) >> 4);
              sep::mma_bf16_ss(tmem + cs, dQ + oq, dK + okv, id_s, kk > 0 ? 1u : 0u);
              sep::mma_bf16_ss(tmem + cs + 64, dO + oq, dV + okv, id_s, kk > 0 ? 1u : 0u);
            }
            sep::mma_commit(&bars.s_full[gu & 1]);
            if (u == nunit - 1) sep::mma_commit(&bars.q_free[qbuf]);  // the item's Q, dO are read
          }
          if (u >= 1) {
            const uint32_t w = U + u - 1;
            const int wst = w % kNst;
            if (!sep::mbar_wait(&bars.p_full[w & 1], (w >> 1) & 1, abort, p.err) ||
                (u == 1 && I >= 2 && !sep::mbar_wait(&bars.acc_free[abuf], ((I - 2) >> 1) & 1, abort, p.err))) {
              ok = false;
              break;
            }
            sep::tc_fence_after();
            const uint64_t dKmn = sep::smem_desc_sw128(sb_ + Sm::RING + wst * Sm::STAGE, kT64);
            const uint32_t cs = 128u * (w & 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t off = static_cast<uint64_t>(kk * (2048 >> 4));
              sep::mma_bf16_ts(tmem + cdq, tmem + unit_acol(cs, kk), dKmn + off, id_o,
                               (u > 1 || kk > 0) ? 1u : 0u);
            }
            sep::mma_commit(&bars.st_free[wst]);  // the stage may be refilled
          }
        }
        if (!ok) break;
        sep::mma_commit(&bars.fin[abuf]);
        U += nunit;
      }
      sep::mma_commit(&bars.drain);
      int keep = 0;
      sep::mbar_wait(&bars.drain, 0, &keep, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ loads (warp 9)
    // Per item: its Q and dO once their buffer is free; per unit: the copies
    // once its stage is free, then the global-flag words of a window unit,
    // then the 32 arrivals that complete the stage with its bytes.
    uint32_t U = 0, I = 0;
    uint32_t issued_u = 0, issued_i = 0;
    bool ok = true;
    QItem cur = blockIdx.x < nitems ? q_item(p, blockIdx.x) : QItem{};
    for (int ii = blockIdx.x; ii < nitems && ok; ii += gridDim.x, ++I) {
      const QItem it = cur;
      cur = ii + static_cast<int>(gridDim.x) < nitems ? q_item(p, ii + gridDim.x) : cur;
      const int nunit = it.nunit;
      const int qbuf = I % QB;
      const int64_t kvrow0 = (static_cast<int64_t>(it.b) * p.Hkv + it.h / G) * S;
      const uint8_t* fl = p.is_sep + static_cast<int64_t>(it.b) * S;
      bool go = true;
      if (lane == 0) {
        if (I >= QB) go = sep::mbar_wait(&bars.q_free[qbuf], ((I - QB) / QB) & 1, abort, p.err);
        if (go) {
          const int32_t row = static_cast<int32_t>((static_cast<int64_t>(it.b) * p.Hq + it.h) * S + it.t * TBQ);
          sep::mbar_arrive_expect_tx(&bars.q_full[qbuf], Sm::QSZ);
          load_tile128<D>(smem + qbuf * Sm::QSZ, &map_q, row, &bars.q_full[qbuf]);
          load_tile128<D>(smem + qbuf * Sm::QSZ + NB * kT128, &map_do, row, &bars.q_full[qbuf]);
          load_tile128<D>(smem + qbuf * Sm::QSZ + 2 * NB * kT128, &map_o, row, &bars.q_full[qbuf]);
        }
      }
      if (!__shfl_sync(0xffffffffu, go, 0)) break;
      issued_i = I + 1;
      for (int u = 0; u < nunit; ++u) {
        const uint32_t gu = U + u;
        const int st = gu % kNst;
        const bool win = (u >> 1) >= it.nbg;
        const int key0 = unit_key(it, u);
        bool f[2];  // global flags of keys lane, lane + 32 (loads in flight during the wait)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int q = key0 + lane + 32 * m;
          f[m] = win && q <= it.qlast && (q < p.a || fl[q] != 0);
        }
        if (lane == 0) {
          if (gu >= kNst) go = sep::mbar_wait(&bars.st_free[st], ((gu / kNst) - 1) & 1, abort, p.err);
          if (go) {
            uint8_t* dst = smem + Sm::RING + st * Sm::STAGE;
            const int32_t row = static_cast<int32_t>(kvrow0 + key0);
            mbar_expect_tx(&bars.st_full[st], Sm::STAGE);
#pragma unroll
            for (int c = 0; c < NB; ++c) {
              sep::tma_load_2d(dst + c * kT64, win ? &map_k : &map_kc, 64 * c, row, &bars.st_full[st]);
              sep::tma_load_2d(dst + (NB + c) * kT64, win ? &map_v : &map_vc, 64 * c, row, &bars.st_full[st]);
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, go, 0)) {
          ok = false;
          break;
        }
        issued_u = gu + 1;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const uint32_t w = __ballot_sync(0xffffffffu, f[m]);
          if (lane == m) glb_w[st * 2 + m] = w;
        }
        sep::mbar_arrive(&bars.st_full[st]);
      }
      U += nunit;
    }
    if (lane == 0 && *abort) {
      int dummy = 0;
      for (uint32_t j = issued_i > QB ? issued_i - QB : 0; j < issued_i; ++j)
        sep::mbar_wait(&bars.q_full[j % QB], (j / QB) & 1, &dummy, nullptr);
      for (uint32_t g2 = issued_u > kNst ? issued_u - kNst : 0; g2 < issued_u; ++g2)
        sep::mbar_wait(&bars.st_full[g2 % kNst], (g2 / kNst) & 1, &dummy, nullptr);
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

// Workspace: delta [B, Hq, S] fp32; fp32 dK and dV rows of the compact
// global-key lists [B, Hkv, S, D] each; the compact bf16 K and V copies
// [B, Hkv, S, D] each; the global-key work items (at most B x ceil(S/128) x
// ceil(ceil(S/128)/chunk_tiles) x Hkv global items and B x ceil(S/128) x
// Hkv window items, pairs of int32) after their count and the per-sequence
// offsets.
struct BwdWs {
  size_t delta, dk, dv, kc, vc, items;
  size_t total() const { return delta + dk + dv + kc + vc + items; }
};
BwdWs bwd_ws(int B, int Hq, int Hkv, int S, int D) {
  auto r256 = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t nwin = (static_cast<size_t>(S) + TBK - 1) / TBK;
  const int ct = D == 64 ? chunk_tiles<64>() : chunk_tiles<128>();
  const size_t nchunk = (nwin + ct - 1) / ct;
  BwdWs w;
  w.delta = r256(static_cast<size_t>(B) * Hq * S * 4);
  w.dk = r256(static_cast<size_t>(B) * Hkv * S * D * 4);
  w.dv = w.dk;
  w.kc = r256(static_cast<size_t>(B) * Hkv * S * D * 2);
  w.vc = w.kc;
  w.items = r256(4 + static_cast<size_t>(B) * 4) +
            r256(static_cast<size_t>(B) * Hkv * nwin * (nchunk + 1) * 8);
  return w;
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
int launch_bwd(BwdParams p, const void* out, void* dq, void* dk, void* dv, void* ws,
               cudaStream_t st) {
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(k_bwd_kv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             KvSmem<D>::BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(k_bwd_q<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QSmem<D>::BYTES) != cudaSuccess)
      return SEP_ECUDA;
    attr_done[dev] = true;
  }
  const BwdWs w = bwd_ws(p.B, p.Hq, p.Hkv, p.S, D);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* delta = reinterpret_cast<float*>(base);
  p.delta = delta;
  p.dk_acc = reinterpret_cast<float*>(base + w.delta);
  p.dv_acc = reinterpret_cast<float*>(base + w.delta + w.dk);
  __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(base + w.delta + w.dk + w.dv);
  __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(base + w.delta + w.dk + w.dv + w.kc);
  p.item_count = reinterpret_cast<int32_t*>(base + w.delta + w.dk + w.dv + w.kc + w.vc);
  p.items = reinterpret_cast<int2*>(base + w.delta + w.dk + w.dv + w.kc + w.vc +
                                    (4 + static_cast<size_t>(p.B) * 4 + 255) / 256 * 256);
  p.nwin = (p.S + TBK - 1) / TBK;
  p.ctiles = chunk_tiles<D>();
  p.nchunk = (p.nwin + p.ctiles - 1) / p.ctiles;
  const int64_t qrows = static_cast<int64_t>(p.B) * p.Hq * p.S;
  const int64_t krows = static_cast<int64_t>(p.B) * p.Hkv * p.S;
  if (qrows > 0x7fffffffLL) return SEP_ETOOBIG;
  // 128-row boxes for the operands a CTA keeps (K, V of the key-centric
  // kernel; Q, dO of the query-centric one), 64-row boxes for the ring units
  CUtensorMap mq, mdo, mo, mk, mv, mkc, mvc, uq, udo, uk, uv, ukc, uvc;
  if (!sep::make_rows_map(&mq, p.q, qrows, D, TBQ) || !sep::make_rows_map(&mdo, p.dout, qrows, D, TBQ) ||
      !sep::make_rows_map(&mo, out, qrows, D, TBQ) ||
      !sep::make_rows_map(&mk, p.k, krows, D, TBK) || !sep::make_rows_map(&mv, p.v, krows, D, TBK) ||
      !sep::make_rows_map(&mkc, kc, krows, D, TBK) || !sep::make_rows_map(&mvc, vc, krows, D, TBK) ||
      !sep::make_rows_map(&uq, p.q, qrows, D, 64) || !sep::make_rows_map(&udo, p.dout, qrows, D, 64) ||
      !sep::make_rows_map(&uk, p.k, krows, D, 64) || !sep::make_rows_map(&uv, p.v, krows, D, 64) ||
      !sep::make_rows_map(&ukc, kc, krows, D, 64) || !sep::make_rows_map(&uvc, vc, krows, D, 64))
    return SEP_ECUDA;
  const dim3 rgrid((p.S + 63) / 64, p.Hkv, p.B);
  // Launch chain.  The plan is a plain launch: it starts once all earlier
  // work on the stream has completed.  Every later kernel is a programmatic
  // launch that overlaps the tail of the one before and runs
  // griddepcontrol.wait before it reads any output of this call: k_bwd_prep
  // runs alongside the plan (it reads only the index) and one of its CTAs
  // waits for the plan before it ends, so each wait covers every launch
  // before it.  The plan must stay a plain launch.
  k_bwd_plan<<<1, 32 * kPlanWarps, 0, st>>>(p);
  if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  if (sep::launch_pdl(k_bwd_prep<D>, rgrid, dim3(256), 0, st, p, kc, vc) != cudaSuccess)
    return SEP_ECUDA;
  // persistent: one CTA per SM (shared memory and TMEM hold one)
  const int sms = num_sms();
  // dQ and delta first, then dK and dV (which read delta)
  const int64_t qitems = static_cast<int64_t>(p.B) * p.Hq * ((p.S + TBQ - 1) / TBQ);
  if (sep::launch_pdl(k_bwd_q<D>, dim3(static_cast<unsigned>(qitems < sms ? qitems : sms)),
                     dim3(kTcThreads), QSmem<D>::BYTES, st, p, mq, mdo, mo, uk, uv, ukc, uvc,
                     static_cast<__nv_bfloat16*>(dq)) != cudaSuccess)
    return SEP_ECUDA;
  if (sep::launch_pdl(k_bwd_kv<D>, dim3(sms), dim3(kTcThreads), KvSmem<D>::BYTES, st, p, uq, udo, mk,
                     mv, mkc, mvc, static_cast<__nv_bfloat16*>(dk),
                     static_cast<__nv_bfloat16*>(dv)) != cudaSuccess)
    return SEP_ECUDA;
  if (sep::launch_pdl(k_bwd_scatter<D>, rgrid, dim3(256), 0, st, p,
                     p.scale_log2 / 1.44269504088896340736f, static_cast<__nv_bfloat16*>(dk),
                     static_cast<__nv_bfloat16*>(dv)) != cudaSuccess)
    return SEP_ECUDA;
  return sep::launch_status();
}

}  // namespace

extern "C" size_t sep_attn_backward_workspace(int B, int Hq, int Hkv, int S, int D) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || Hq % Hkv != 0 || (D != 64 && D != 128)) return 0;
  return bwd_ws(B, Hq, Hkv, S, D).total();
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
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return D == 64 ? launch_bwd<64>(p, out, dq, dk, dv, workspace, st)
                 : launch_bwd<128>(p, out, dq, dk, dv, workspace, st);
}
