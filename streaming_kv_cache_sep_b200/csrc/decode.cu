// Decode attention of the newest token over the SepCache (split-K, GQA-aware).
//
// The cache keeps only the initial, separator, past-window and local-window
// rows, so a decode step reads len[b] <= a + s + past + w K/V rows per
// (sequence, kv head) (jieyibu.net explainer, section 1.3: fewer KV pairs to
// load).  The kernel is bound by HBM bandwidth and by its latency chain:
//   * grid (split, kv head, sequence); a CTA takes 64 consecutive rows of one
//     (b, kv head) and pulls them into shared memory with two bulk copies
//     (K and V, one mbarrier), so each byte is read from HBM once per step;
//   * the G = Hq/Hkv query heads of the group share every K/V row; a warp
//     scores four rows at a time (eight lanes per row, each lane 8 or 16
//     dims), so a row costs three shuffle levels instead of five;
//   * each CTA produces an unnormalised partial (max, sum, G x D output).
//     With at most 8 splits the splits of a (b, kv head) form one
//     thread-block cluster and merge the partials through distributed shared
//     memory; otherwise they go through the workspace and the last CTA to
//     finish (an atomic ticket, no waiting) merges them;
//   * launched as a programmatic dependent launch: the grid may start while
//     the previous kernel on the stream drains, and waits for it before its
//     first global read.
#include <cooperative_groups.h>
#include <string.h>

#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace {

constexpr int ROWS = 64;  // rows per split
constexpr int kThreads = 128;
constexpr int kMaxClusterSplits = 8;

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// 8 consecutive elements (16-byte aligned) as floats.
__device__ __forceinline__ void ld8(const __nv_bfloat16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void ld8(const float* p, float* x) {
  const float4 a = reinterpret_cast<const float4*>(p)[0];
  const float4 b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }

struct DecodeParams {
  const void* q;
  const void* kc;
  const void* vc;
  const int32_t* counts;
  const int32_t* plan;  // [B][cap + header] this step's plan (fused step only)
  const void* k_new;    // [B][Hkv][D] (fused step only)
  const void* v_new;
  void* out;
  float* lse;
  float* part_ml;  // [B][Hq][nsplit][2]
  float* part_o;   // [B][Hq][nsplit][D]
  int32_t* ticket; // [B][Hkv]
  int32_t* err;
  int layer, layers, B, Hq, Hkv, cap, nsplit;
  int early;  // fused step of layer >= 1: cache reads may precede the grid-dependency wait
  float scale_log2;
  // positional-encoding shifting: keys are stored un-encoded and encoded at
  // their slot in the cache, q at the newest slot len - 1; rope[r][i] =
  // (cos, sin) of r * theta^(-2i/D), rope_rows >= max(cap, 65).  null: off
  const float* rope;
  int rope_rows;
  // mask-based generation over a full history (null prefix: the cache path).
  // kc, vc: k, v [B][Hkv][S][D]; the query is token T - 1; its kept set is
  // [0, min(a, lo)), the separators in [min(a, lo), lo) (idx[b][prefix[b][.]]),
  // and the window [lo, T), lo = max(0, T - n)
  const int32_t* prefix;  // [B][S + 1]
  const int32_t* idx;     // [B][S]
  int S, T, a, n;
};

// The kept rows of the generating token: count and the history row of the
// i-th kept row (ascending positions).
struct GenRows {
  int lo, a0, pa, nsep, len;
  const int32_t* ix;
  __device__ __forceinline__ GenRows(const DecodeParams& p, int b) {
    lo = p.T - p.n > 0 ? p.T - p.n : 0;
    a0 = p.a < lo ? p.a : lo;
    const int32_t* pre = p.prefix + static_cast<int64_t>(b) * (p.S + 1);
    pa = pre[a0];
    nsep = pre[lo] - pa;
    len = a0 + nsep + (p.T - lo);
    ix = p.idx + static_cast<int64_t>(b) * p.S;
  }
  __device__ __forceinline__ int row(int i) const {
    return i < a0 ? i : (i < a0 + nsep ? ix[pa + i - a0] : lo + (i - a0 - nsep));
  }
};

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
// arrive on `bar` once this thread's earlier cp.async copies have landed
// (the barrier's expected count includes this arrival)
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(sep::smem_u32(bar))
               : "memory");
}

// The last part of a split: its unnormalised partial (po, sm = max, sl = sum,
// in this CTA's shared memory, rows with no keys at -inf / 0) is merged with
// the other splits of the (b, kv head) and written out.  Returns true in
// exactly one CTA of the (b, kv head), at a point where every split has
// finished reading its K/V rows (the CTA that may then move rows in place).
template <typename T, int D, int G, bool CLUSTER, int NCL = kMaxClusterSplits>
__device__ __forceinline__ bool decode_finish(const DecodeParams& p, float (*po)[D], float* sm,
                                              float* sl, int nsplit_b, int split, int b, int g) {
  __shared__ int is_last;
  __shared__ float Ms[G], Ls[G];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  T* out = static_cast<T*>(p.out);
  const int hq0 = g * G;
  if (nsplit_b == 1) {
    if (split == 0) {
      for (int e = threadIdx.x; e < G * D; e += kThreads) {
        const int h = e / D, d = e % D;
        out[(static_cast<int64_t>(b) * p.Hq + hq0 + h) * D + d] = from_f<T>(po[h][d] / sl[h]);
      }
      if (p.lse && threadIdx.x < G)
        p.lse[static_cast<int64_t>(b) * p.Hq + hq0 + threadIdx.x] =
            (sm[threadIdx.x] + log2f(sl[threadIdx.x])) * 0.69314718055994530942f;
    }
    if (CLUSTER) {
      cg::this_cluster().sync();
      cg::this_cluster().sync();
    }
    return split == 0;
  }
  if (CLUSTER) {
    // after the cluster barrier CTA `split` merges outputs
    // [split*G*D/NCL, (split+1)*G*D/NCL) from the shared memory of all splits
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();
    constexpr int PER = G * D / NCL;
    for (int e = threadIdx.x; e < PER; e += blockDim.x) {
      const int idx = split * PER + e;
      const int h = idx / D, d = idx % D;
      float M = -INFINITY;
      float mk[NCL], lk[NCL], ok[NCL];
#pragma unroll
      for (int k = 0; k < NCL; ++k) {
        const bool in = k < nsplit_b;
        mk[k] = in ? *cl.map_shared_rank(&sm[h], k) : -INFINITY;
        lk[k] = in ? *cl.map_shared_rank(&sl[h], k) : 0.f;
        ok[k] = in ? *cl.map_shared_rank(&po[h][d], k) : 0.f;
        M = fmaxf(M, mk[k]);
      }
      float L = 0.f, acc = 0.f;
#pragma unroll
      for (int k = 0; k < NCL; ++k) {
        const float w = k < nsplit_b ? exp2f(mk[k] - M) : 0.f;
        L += lk[k] * w;
        acc += ok[k] * w;
      }
      out[(static_cast<int64_t>(b) * p.Hq + hq0 + h) * D + d] = from_f<T>(acc / L);
      if (p.lse && d == 0)
        p.lse[static_cast<int64_t>(b) * p.Hq + hq0 + h] = (M + log2f(L)) * 0.69314718055994530942f;
    }
    cl.sync();  // keep this CTA's partial alive until every reader is done
    return split == 0;
  }
  if (split >= nsplit_b) return false;
  // write this split's partial to the workspace
  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int h = e / D, d = e % D;
    p.part_o[((static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit + split) * D + d] = po[h][d];
  }
  if (threadIdx.x < G) {
    float* ml = p.part_ml + ((static_cast<int64_t>(b) * p.Hq + hq0 + threadIdx.x) * p.nsplit + split) * 2;
    ml[0] = sm[threadIdx.x];
    ml[1] = sl[threadIdx.x];
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t* tk = p.ticket + static_cast<int64_t>(b) * p.Hkv + g;
    const int prev = atomicAdd(tk, 1);
    is_last = prev == nsplit_b - 1;
    if (is_last) atomicExch(tk, 0);  // ready for the next call
  }
  __syncthreads();
  if (!is_last) return false;
  __threadfence();
  // merge the partials of every split of this (b, kv head).  Loads that do
  // not depend on each other are issued together: one lane per split for the
  // (max, sum) pairs, then eight splits at a time for the output rows.
  for (int h = warp; h < G; h += 4) {
    const float* ml = p.part_ml + (static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit * 2;
    float M = -INFINITY;
    for (int s = lane; s < nsplit_b; s += 32) M = fmaxf(M, __ldcg(ml + 2 * s));
    for (int o2 = 16; o2; o2 >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o2));
    float Lsum = 0.f;
    for (int s = lane; s < nsplit_b; s += 32) Lsum += __ldcg(ml + 2 * s + 1) * exp2f(__ldcg(ml + 2 * s) - M);
    for (int o2 = 16; o2; o2 >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o2);
    if (lane == 0) {
      Ms[h] = M;
      Ls[h] = Lsum;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int h = e / D, d = e % D;
    const float* ml = p.part_ml + (static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit * 2;
    const float* pp = p.part_o + (static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit * D;
    const float M = Ms[h];
    float acc = 0.f;
    for (int s0 = 0; s0 < nsplit_b; s0 += 8) {
      float ov[8], mv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s0 + u;
        const bool in = s < nsplit_b;
        ov[u] = in ? __ldcg(pp + s * D + d) : 0.f;
        mv[u] = in ? __ldcg(ml + 2 * s) : -INFINITY;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) acc += ov[u] * exp2f(mv[u] - M);
    }
    out[(static_cast<int64_t>(b) * p.Hq + hq0 + h) * D + d] = from_f<T>(acc / Ls[h]);
  }
  if (p.lse && threadIdx.x < G)
    p.lse[static_cast<int64_t>(b) * p.Hq + hq0 + threadIdx.x] =
        (Ms[threadIdx.x] + log2f(Ls[threadIdx.x])) * 0.69314718055994530942f;
  return true;
}

// In-place flush of one layer's destination rows [from, len) of one (b, kv
// head), by one CTA of nthreads threads, once every reader of their old
// rows is done: destination row r takes source row plan.src[r] >= r (src
// increasing; the new token, src == slot, from k_new / v_new).  Ascending chunks of `rows` rows staged
// in shared memory (sk, sv), every source of a chunk read before any of its
// destinations is written, so no row is overwritten before it is read.
// Rows with src[r] == r (the initial block, and separators that stay) are
// left alone; the new token's row (src == slot) is always written.
template <typename T, int D>
__device__ __forceinline__ void compact_in_place(const DecodeParams& p, int b, int g, int from,
                                                 int len, int slot, int rows, int nthreads, T* sk,
                                                 T* sv) {
  constexpr int CH = D * static_cast<int>(sizeof(T)) / 16;
  const int32_t* pl = p.plan + static_cast<int64_t>(b) * (p.cap + sep::kCachePlanHdr);
  const int64_t base = (((static_cast<int64_t>(p.layer) * p.B + b) * p.Hkv + g) * p.cap) * D;
  T* const kc = static_cast<T*>(const_cast<void*>(p.kc));
  T* const vc = static_cast<T*>(const_cast<void*>(p.vc));
  const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
  const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
  const int first = pl[3] > from ? pl[3] : from;
  for (int c0 = first; c0 < len; c0 += rows) {
    const int nr = len - c0 < rows ? len - c0 : rows;
    for (int e = threadIdx.x; e < 2 * nr * CH; e += nthreads) {
      const int which = e / (nr * CH), r = (e / CH) % nr, c = e % CH;
      const int src = pl[sep::kCachePlanHdr + c0 + r];
      uint4 val = make_uint4(0, 0, 0, 0);
      if (src == slot) {
        val = (which ? vn : kn)[c];
      } else if (src >= 0 && src < p.cap) {
        val = reinterpret_cast<const uint4*>((which ? vc : kc) + base + static_cast<int64_t>(src) * D)[c];
      }
      reinterpret_cast<uint4*>((which ? sv : sk) + r * D)[c] = val;
    }
    __syncthreads();  // every source of the chunk has been read
    for (int e = threadIdx.x; e < 2 * nr * CH; e += nthreads) {
      const int which = e / (nr * CH), r = (e / CH) % nr, c = e % CH;
      const int src = pl[sep::kCachePlanHdr + c0 + r];
      if (src == c0 + r && src != slot) continue;  // the row stays
      reinterpret_cast<uint4*>((which ? vc : kc) + base + static_cast<int64_t>(c0 + r) * D)[c] =
          reinterpret_cast<const uint4*>((which ? sv : sk) + r * D)[c];
    }
    __syncthreads();
  }
}

// FUSED: one decode step of the layer -- the CTA also writes the new token's
// K/V row and, on a flush step, copies its share of the surviving rows into
// the sequence's other buffer while loading them (see sepcache.cu).
// CLUSTER: the grid's x dimension (the splits) is one cluster.
template <typename T, int D, int G, bool FUSED, bool CLUSTER>
__global__ void __launch_bounds__(kThreads, (G <= 4 ? 5 : 3)) k_decode(const DecodeParams p) {
  constexpr int NI = D / 64;   // 8-element slices per lane: dims 8*c8 + 64*i + e
  constexpr int DPL = 8 * NI;  // dims per lane
  // dynamic: K rows | V rows; the cross-warp reduction reuses the K rows
  extern __shared__ __align__(128) uint8_t dsm[];
  T* sk = reinterpret_cast<T*>(dsm);
  T* sv = sk + ROWS * D;
  float(*red)[G][D] = reinterpret_cast<float(*)[G][D]>(dsm);
  static_assert(sizeof(T) * ROWS * D >= sizeof(float) * 4 * G * D, "reduction must fit in K rows");
  __shared__ float ss[G][ROWS];
  __shared__ float po[G][D];  // this CTA's partial output (cluster merge)
  __shared__ float sm[G], sl[G];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rr = lane >> 3, c8 = lane & 7;  // row of the 4-row group, 8-dim slice

  // wait for the previous kernel on the stream (programmatic dependent launch)
  asm volatile("griddepcontrol.wait;" ::: "memory");

  // metadata: independent loads issued together
  const int32_t* cnt = p.counts + 4 * b;
  const int32_t* pl = p.plan + static_cast<int64_t>(b) * (p.cap + sep::kCachePlanHdr);
  const bool gen = p.prefix != nullptr;  // mask-based generation over k, v
  const int c0 = gen ? 0 : cnt[0], c1 = gen ? 0 : cnt[1], c2 = gen ? 0 : cnt[2], c3 = gen ? 0 : cnt[3];
  const int flush = FUSED ? pl[0] : 0;
  const int slot = FUSED ? pl[1] : -1;
  int len = c0 + c1 + c2 + c3;
  if (gen) len = GenRows(p, b).len;
  if (len < 0 || len > p.cap) len = 0;
  const int r0 = split * ROWS;
  const int nrows = len - r0 < 0 ? 0 : (len - r0 < ROWS ? len - r0 : ROWS);
  if (!CLUSTER && nrows == 0) return;
  const int nsplit_b = (len + ROWS - 1) / ROWS;
  // element offset of row 0 of (layer, b, g)
  const int64_t base = (((static_cast<int64_t>(p.layer) * p.B + b) * p.Hkv + g) * p.cap) * D;
  const int64_t kv_base = base + static_cast<int64_t>(r0) * D;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sep::mbar_init(&bar, 1);
    sep::mbar_fence_init();
  }
  __syncthreads();
  const bool bulk = nrows > 0 && !flush && !gen;
  if (gen && nrows > 0) {
    // the split's kept rows, gathered from k, v [B][Hkv][S][D]
    const GenRows gr(p, b);
    const int64_t hbase = (static_cast<int64_t>(b) * p.Hkv + g) * p.S;
    constexpr int CU = D * static_cast<int>(sizeof(T)) / 16;
    for (int e = threadIdx.x; e < 2 * nrows * CU; e += kThreads) {
      const int which = e / (nrows * CU), r = (e / CU) % nrows, c = e % CU;
      const int64_t hr = hbase + gr.row(r0 + r);
      reinterpret_cast<uint4*>((which ? sv : sk) + r * D)[c] =
          reinterpret_cast<const uint4*>(static_cast<const T*>(which ? p.vc : p.kc) + hr * D)[c];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0 && bulk) {
    const uint32_t bytes = static_cast<uint32_t>(nrows * D * sizeof(T));
    sep::mbar_arrive_expect_tx(&bar, 2 * bytes);
    sep::bulk_load(sk, static_cast<const T*>(p.kc) + kv_base, bytes, &bar);
    sep::bulk_load(sv, static_cast<const T*>(p.vc) + kv_base, bytes, &bar);
  }
  // let the next kernel on the stream begin launching
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // this lane's query slices of the group's heads, pre-scaled (log2 domain)
  const T* qg = static_cast<const T*>(p.q) + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
  float qv[G][DPL];
  const int mq = len > 0 ? len - 1 : 0;  // the newest token's slot
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < NI; ++i) {
      ld8(qg + h * D + 64 * i + 8 * c8, &qv[h][8 * i]);
      if (p.rope) {
        // encode at slot mq: dims d < D/2 pair with d + D/2
        const int d0 = 64 * i + 8 * c8;
        const bool lo = d0 < D / 2;
        const int dp = lo ? d0 + D / 2 : d0 - D / 2;
        float y[8];
        ld8(qg + h * D + dp, y);
        const float* cs = p.rope + static_cast<int64_t>(mq) * D + 2 * (lo ? d0 : dp);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x = qv[h][8 * i + e];
          qv[h][8 * i + e] = lo ? x * cs[2 * e] - y[e] * cs[2 * e + 1] : x * cs[2 * e] + y[e] * cs[2 * e + 1];
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) qv[h][8 * i + e] *= p.scale_log2;
    }
  constexpr int CH = D * static_cast<int>(sizeof(T)) / 16;  // 16-byte chunks per row
  if (FUSED && flush && nrows > 0) {
    // rows of the post-flush layout come from their source rows (the new
    // token from k_new/v_new); the rows move in place only after every split
    // of the (b, kv head) has read its sources (compact_in_place)
    const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
    const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
    for (int e = threadIdx.x; e < 2 * nrows * CH; e += kThreads) {
      const int which = e / (nrows * CH), r = (e / CH) % nrows, c = e % CH;
      const int src = pl[sep::kCachePlanHdr + r0 + r];
      uint4 val = make_uint4(0, 0, 0, 0);
      if (src == slot) {
        val = (which ? vn : kn)[c];
      } else if (src >= 0 && src < p.cap) {
        val = reinterpret_cast<const uint4*>(static_cast<const T*>(which ? p.vc : p.kc) + base +
                                             static_cast<int64_t>(src) * D)[c];
      }
      reinterpret_cast<uint4*>((which ? sv : sk) + r * D)[c] = val;
    }
    __syncthreads();
  } else if (bulk) {
    const bool landed = sep::mbar_wait(&bar, 0, &abort_flag, p.err);
    if (!landed) {  // the copies must land before this CTA's shared memory is reused
      int keep_waiting = 0;
      sep::mbar_wait(&bar, 0, &keep_waiting, nullptr);
    }
    if (FUSED && slot >= r0 && slot < r0 + nrows) {
      // the new token is the last row (no flush): take it from k_new/v_new
      // and store it into the cache
      const int r = slot - r0;
      const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
      const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
      for (int e = threadIdx.x; e < 2 * CH; e += kThreads) {
        const int which = e / CH, c = e % CH;
        const uint4 val = (which ? vn : kn)[c];
        reinterpret_cast<uint4*>((which ? sv : sk) + r * D)[c] = val;
        reinterpret_cast<uint4*>(const_cast<T*>(static_cast<const T*>(which ? p.vc : p.kc)) + kv_base +
                                 static_cast<int64_t>(r) * D)[c] = val;
      }
      __syncthreads();
    }
  }

  if (p.rope) {
    // encode the split's K rows in place at their slots r0 + r (the cache
    // keeps them un-encoded)
    for (int e = threadIdx.x; e < nrows * (D / 2); e += kThreads) {
      const int r = e / (D / 2), i = e % (D / 2);
      const float2 cs = reinterpret_cast<const float2*>(p.rope)[static_cast<int64_t>(r0 + r) * (D / 2) + i];
      const float x = to_f(sk[r * D + i]), y = to_f(sk[r * D + i + D / 2]);
      sk[r * D + i] = from_f<T>(x * cs.x - y * cs.y);
      sk[r * D + i + D / 2] = from_f<T>(y * cs.x + x * cs.y);
    }
    __syncthreads();
  }

  // scores: warp w takes 4-row groups w, w+4, ...; lane (rr, c8) covers dims
  // 8*c8 + 64*i + [0, 8) of row 4*group + rr
  for (int r4 = 4 * warp; r4 < nrows; r4 += 16) {
    const int r = r4 + rr;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
    if (r < nrows) {
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        float x[8];
        ld8(sk + r * D + 64 * i + 8 * c8, x);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[h] = fmaf(qv[h][8 * i + e], x[e], acc[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
    if (r < nrows) {
#pragma unroll
      for (int h = 0; h < G; ++h)
        if (c8 == (h & 7)) ss[h][r] = acc[h];
    }
  }
  __syncthreads();
  // per-head softmax over this split's rows
  for (int h = warp; h < G; h += 4) {
    float m = -INFINITY;
    for (int r = lane; r < nrows; r += 32) m = fmaxf(m, ss[h][r]);
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int r = lane; r < nrows; r += 32) {
      const float e = exp2f(ss[h][r] - m);
      ss[h][r] = e;
      l += e;
    }
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      sm[h] = m;
      sl[h] = l;
    }
  }
  __syncthreads();
  // P V: lane (rr, c8) accumulates its dims over rows rr, rr+4, ... of the
  // warp's groups; then rows of a lane slice and warps are summed
  float o[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[h][e] = 0.f;
  for (int r4 = 4 * warp; r4 < nrows; r4 += 16) {
    const int r = r4 + rr;
    if (r < nrows) {
      float pr[G];
#pragma unroll
      for (int h = 0; h < G; ++h) pr[h] = ss[h][r];
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        float x[8];
        ld8(sv + r * D + 64 * i + 8 * c8, x);
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int e = 0; e < 8; ++e) o[h][8 * i + e] = fmaf(pr[h], x[e], o[h][8 * i + e]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 8);
      o[h][e] += __shfl_xor_sync(0xffffffffu, o[h][e], 16);
    }
  __syncthreads();  // K rows are no longer read: reuse them for the reduction
  if (rr == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int i = 0; i < NI; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) red[warp][h][64 * i + 8 * c8 + e] = o[h][8 * i + e];
  }
  __syncthreads();

  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int h = e / D, d = e % D;
    po[h][d] = nrows > 0 ? red[0][h][d] + red[1][h][d] + red[2][h][d] + red[3][h][d] : 0.f;
  }
  if (threadIdx.x < G && nrows == 0) {
    sm[threadIdx.x] = -INFINITY;
    sl[threadIdx.x] = 0.f;
  }
  __syncthreads();
  const bool owner = decode_finish<T, D, G, CLUSTER>(p, po, sm, sl, nsplit_b, split, b, g);
  if (FUSED && flush && owner) {
    // every split has read its sources: move the rows in place
    __syncthreads();
    compact_in_place<T, D>(p, b, g, 0, len, slot, ROWS, kThreads, sk, sv);
  }
}

// ---- warp-level tensor-core helpers (bf16 in, fp32 accumulate)
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
// Transpose of an 8x8 b16 matrix held one 32-bit pair per lane (lane t:
// row t/4, columns 2(t%4), 2(t%4)+1), returned in the same layout.
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
// c (16x8 fp32) += a (16x16 bf16, row-major fragment) * b (16x8 bf16, col fragment)
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16 decode on warp-level tensor cores, streamed by the tensor-copy
// engine.  The rows of a (b, kv head) are split between the NCL CTAs of a
// cluster (about len/NCL rows each).  One producer thread streams a CTA's
// rows in 64-row chunks through a shared-memory ring: per chunk and tensor,
// D/64 tensor-map tiles of 64 rows x 128 bytes, written 128-byte swizzled
// (16-byte unit u of row r lands at unit u ^ (r & 7)), so a chunk is
// 2 * D/64 copy requests of 8 KB and the ldmatrix reads hit eight different
// bank groups.  When a CTA's rows fit the ring (len <= NCL * stages * 64)
// all its copies start at once.  Each of the four consumer warps owns 16
// rows of every chunk and keeps its own online softmax in registers, with
// the keys as the 16 rows of the tensor-core tile:
//   S^T = K Q^T (A = K rows, B = Q^T: the G query heads as the 8 columns);
//   a head's reference max moves only when a score exceeds it by 2^8;
//   P^T reaches the B operand by an in-register 8x8 transpose (movmatrix);
//   O^T += V^T P^T (A = V^T by ldmatrix.trans).
// No CTA-wide barrier inside the loop.  At the end each CTA merges 1/NCL of
// the D x G outputs: every warp sends its partial for each slice to the CTA
// that merges it with asynchronous remote stores that complete on that
// CTA's mbarrier by byte count, so no sender waits for an acknowledgement.
constexpr int kPipeCluster = 2;
constexpr int kPipeThreads = 160;  // 4 consumer warps + 1 producer warp
constexpr int kTileBytes = ROWS * 128;
constexpr float kLazyLog2 = 8.f;  // reference-max slack (log2 units) before a rescale

template <int D>
__host__ __device__ constexpr int pipe_stage_bytes() {
  return 2 * (D / 64) * kTileBytes;
}
// ring stages: three, except where two CTAs per SM would not fit
template <int D, int G>
__host__ __device__ constexpr int pipe_stages() {
  return D * G >= 1024 ? 2 : 3;
}
// the ring, then the partials this CTA merges ([NCL][4 warps][D/NCL x G] fp32)
template <int D, int G>
__host__ __device__ constexpr int pipe_smem_bytes() {
  return pipe_stages<D, G>() * pipe_stage_bytes<D>() + 4 * G * D * 4 + 1024;  // + alignment slack
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

// Turn the bf16 pairs lo = (x_f, x_f+1) and hi = (x_{f+D/2}, x_{f+1+D/2})
// by the angles with cosines c = (c_f, c_f+1) and sines s: x_f + j x_{f+D/2}
// times exp(j phi), in fp32 (packed pairs).  The results go out as tf32
// operands (l: dims f, f+1; h: dims f+D/2, f+1+D/2): the fp32 bit patterns
// as they are, of which the tensor core reads the top 19 bits (sign, 8-bit
// exponent, 10-bit fraction), so the encoded scores carry less than 2^-10
// relative error per operand instead of bf16's 2^-9.
__device__ __forceinline__ void rope_tf32(uint32_t lo, uint32_t hi, float2 c, float2 s,
                                          uint32_t (&l)[2], uint32_t (&h)[2]) {
  const float2 a = make_float2(__uint_as_float(lo << 16), __uint_as_float(lo & 0xffff0000u));
  const float2 b = make_float2(__uint_as_float(hi << 16), __uint_as_float(hi & 0xffff0000u));
  const float2 lv = fsub2(fmul2(a, c), fmul2(b, s));
  const float2 hv = sep::ffma2(a, s, fmul2(b, c));
  l[0] = __float_as_uint(lv.x);
  l[1] = __float_as_uint(lv.y);
  h[0] = __float_as_uint(hv.x);
  h[1] = __float_as_uint(hv.y);
}
// (c, s) times (mc, ms) as complex numbers, two frequencies at once
__device__ __forceinline__ void cturn(float2& c, float2& s, float2 mc, float2 ms) {
  const float2 nc = fsub2(fmul2(c, mc), fmul2(s, ms));
  s = sep::ffma2(c, ms, fmul2(s, mc));
  c = nc;
}
// c (16x8 fp32) += a (16x8 tf32, row-major fragment) * b (8x8 tf32, col fragment)
__device__ __forceinline__ void mma1688(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte offset of (row r, element d) in one tensor's D/64 swizzled tiles.
__device__ __forceinline__ uint32_t swz(int r, int d) {
  return static_cast<uint32_t>((d >> 6) * kTileBytes + r * 128 +
                               ((((d >> 3) & 7) ^ (r & 7)) << 4) + (d & 7) * 2);
}

template <int D, int G, bool FUSED, bool ROPE, bool GATHER>
__global__ void __launch_bounds__(kPipeThreads, 2)
    k_decode_pipe(const DecodeParams p, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v) {
  static_assert(G <= 8, "at most 8 query heads per kv head");
  using T = __nv_bfloat16;
  constexpr int NCL = kPipeCluster;
  constexpr int kPipeStages = pipe_stages<D, G>();
  constexpr int CH = D / 8;   // 16-byte units per row
  constexpr int DT = D / 16;  // 16-dim tiles of the output
  constexpr int NB = D / 64;  // tiles per chunk and tensor
  constexpr int SB = pipe_stage_bytes<D>();
  constexpr int DQ = D / NCL;   // dims merged by each CTA
  constexpr int PART = DQ * G;  // one warp's partial for one CTA's slice, [DQ][G]
  // bytes that reach each CTA's merge barrier: NCL ranks x 4 warps x
  // (partial + max and sum per head)
  constexpr uint32_t kMergeBytes = NCL * 4 * (PART + 2 * G) * 4;
  extern __shared__ uint8_t dsm_raw[];
  // the swizzle pattern repeats every 1024 bytes: tiles start on that boundary
  uint8_t* const ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* const recv_o = reinterpret_cast<float*>(ring + kPipeStages * SB);  // [NCL][4][PART]
  __shared__ float rm[NCL][4][G], rl[NCL][4][G];  // every warp's running max (log2) and sum
  // rotary turns by 8 and by 64 slots: cosines and sines per frequency
  __shared__ __align__(16) float rope_c[2][ROPE ? D / 2 : 2], rope_s[2][ROPE ? D / 2 : 2];
  __shared__ __align__(8) uint64_t full[kPipeStages], empty[kPipeStages], mrg;
  __shared__ int abort_flag;

  const int rank = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int st = 0; st < kPipeStages; ++st) {
      sep::mbar_init(&full[st], GATHER ? 32 : 1);  // gathers: one arrival per producer lane
      sep::mbar_init(&empty[st], 4);
    }
    sep::mbar_init(&mrg, 1);
    sep::mbar_fence_init();
    sep::mbar_arrive_expect_tx(&mrg, kMergeBytes);  // completes once every partial is here
    if constexpr (!GATHER) {
      sep::tma_prefetch_desc(&map_k);
      sep::tma_prefetch_desc(&map_v);
    }
    // let the next grid on the stream launch now: its CTAs take SM slots as
    // soon as ours retire and start their copies while ours drain (its own
    // grid-dependency wait still orders it after this grid)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  // completes long before the first remote store (after the chunk loop):
  // every CTA's barriers are initialised by then
  sep::cluster_arrive_relaxed();
  // With p.early (fused step, layer >= 1) the cache metadata (counts and
  // plan) and this layer's rows are read before waiting on the previous
  // grid; q, k_new, v_new and every store still come after the wait.  This
  // is safe because of how the step is ordered, not because of distance in
  // the stream: the step's bookkeeping kernel (k_cache_advance, launched
  // with the layer-0 call) is a plain launch WITHOUT programmatic stream
  // serialization, so it starts only after every kernel of the previous step
  // has completed (each waits on its predecessor before it ends), and the
  // layer-0 decode, which does wait, starts only after it.  A grid of this
  // step at layer >= 1 can start only once layer 0 has started, so the
  // metadata it reads is this step's, and the rows of this layer were last
  // written by this layer's launch of the previous step, which has ended.
  // If the bookkeeping launch ever became a programmatic launch, these reads
  // would race with the previous step's layers.
  if (!p.early) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int32_t* pl = FUSED ? p.plan + static_cast<int64_t>(b) * (p.cap + sep::kCachePlanHdr) : nullptr;
  int len;
  if constexpr (GATHER) {
    len = GenRows(p, b).len;
  } else {
    const int32_t* cnt = p.counts + 4 * b;
    len = cnt[0] + cnt[1] + cnt[2] + cnt[3];
  }
  const int flush = FUSED ? pl[0] : 0;
  const int slot = FUSED ? pl[1] : -1;
  if (len < 0 || len > p.cap) len = 0;
  const int per = ((len + NCL - 1) / NCL + 15) / 16 * 16;  // rows per CTA (multiple of 16)
  const int rs = rank * per < len ? rank * per : len;
  const int re = rs + per < len ? rs + per : len;
  const int nchunks = (re - rs + ROWS - 1) / ROWS;
  // first row of this (layer, b, kv head) in the [rows, D] view (gathers:
  // first row of (b, kv head) in the [B * Hkv * S, D] view of k, v)
  const int64_t row0 = GATHER ? (static_cast<int64_t>(b) * p.Hkv + g) * p.S
                              : ((static_cast<int64_t>(p.layer) * p.B + b) * p.Hkv + g) * p.cap;
  T* const kc = static_cast<T*>(const_cast<void*>(p.kc));
  T* const vc = static_cast<T*>(const_cast<void*>(p.vc));
  __syncthreads();

  int issued = 0;  // producer: chunks whose copies were started
  // With more chunks than ring stages, the last (shortest) chunk is loaded
  // first: its stage is released almost at once, so the copy of the chunk
  // that has to wait for a free stage starts about one chunk earlier.  Flush
  // steps keep the ascending order (the in-place moves rely on it), and so
  // do the rotary and gather forms (their row state advances chunk by chunk).
  const bool tail_first = !ROPE && !GATHER && !(FUSED && flush) && nchunks > kPipeStages;
  auto chunk_of = [&](int ci) -> int { return tail_first ? (ci == 0 ? nchunks - 1 : ci - 1) : ci; };
  // consumer state.  O^T tiles: o[dt] holds dims 16dt + gq (+8) x heads
  // 2tq, 2tq + 1; the reference max of those two heads (equal across the
  // lanes of a column) and this lane's share of their sums.
  float o[DT][4];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int dt = 0; dt < DT; ++dt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[dt][e] = 0.f;

  if (warp == 4) {
    // ---------------------------------------------------------- producer
    // gathers: the history rows of the lane's two rows of the next chunk,
    // looked up one chunk ahead so the index loads overlap the copies
    int hn[2] = {-1, -1};
    if constexpr (GATHER) {
      const GenRows gr(p, b);
      const int nr0 = re - rs < ROWS ? re - rs : ROWS;
#pragma unroll
      for (int u = 0; u < 2; ++u) hn[u] = 32 * u + lane < nr0 ? gr.row(rs + 32 * u + lane) : -1;
    }
    for (int ci = 0; ci < nchunks; ++ci) {
      const int c = chunk_of(ci);
      const int st = ci % kPipeStages;
      const int r0 = rs + c * ROWS;
      const int nr = re - r0 < ROWS ? re - r0 : ROWS;
      uint8_t* const kt = ring + st * SB;
      uint8_t* const vt = kt + NB * kTileBytes;
      if (ci >= kPipeStages &&
          !__all_sync(0xffffffffu, sep::mbar_wait(&empty[st], ((ci / kPipeStages) - 1) & 1, &abort_flag, p.err)))
        break;
      if constexpr (GATHER) {
        // the chunk's kept rows by 16-byte copies: CH lanes per row (one
        // 256- or 128-byte row segment per instruction group), rows past the
        // chunk's end zero-filled; each lane then arrives on the stage's
        // barrier once its copies have landed
        const GenRows gr(p, b);
        const int hr[2] = {hn[0], hn[1]};
        {
          const int r1 = r0 + ROWS, nr1 = re - r1 < ROWS ? re - r1 : ROWS;
#pragma unroll
          for (int u = 0; u < 2; ++u) hn[u] = 32 * u + lane < nr1 ? gr.row(r1 + 32 * u + lane) : -1;
        }
        constexpr int RPI = 32 / CH;  // rows per warp instruction
        const uint32_t kts = sep::smem_u32(kt), vts = sep::smem_u32(vt);
#pragma unroll 4
        for (int it = 0; it < ROWS / RPI; ++it) {
          const int q = it * RPI + lane / CH, cc = lane % CH;
          const int src = __shfl_sync(0xffffffffu, (it * RPI) >> 5 ? hr[1] : hr[0], q & 31);
          const int64_t off = (row0 + (src < 0 ? 0 : src)) * D + 8 * cc;
          const uint32_t nb = src < 0 ? 0u : 16u;
          cp_async16(kts + swz(q, 8 * cc), kc + off, nb);
          cp_async16(vts + swz(q, 8 * cc), vc + off, nb);
        }
        cp_async_arrive(&full[st]);
      } else if (FUSED && flush) {
        // rows of the post-flush layout come from their source rows (the
        // new token from k_new/v_new).  The first CTA of the pair also
        // stores each row at its destination, in place: its destinations
        // lie below every source of the second CTA and below the sources of
        // its own later chunks.  The second CTA's destinations may be the
        // first one's sources, so it moves its rows after the merge.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
        const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
        for (int e = lane; e < 2 * nr * CH; e += 32) {
          const int which = e / (nr * CH), r = (e / CH) % nr, cc = e % CH;
          const int src = pl[sep::kCachePlanHdr + r0 + r];
          uint4 val = make_uint4(0, 0, 0, 0);
          if (src == slot) {
            val = (which ? vn : kn)[cc];
          } else if (src >= 0 && src < p.cap) {
            val = reinterpret_cast<const uint4*>((which ? vc : kc) + (row0 + src) * D)[cc];
          }
          *reinterpret_cast<uint4*>((which ? vt : kt) + swz(r, 8 * cc)) = val;
          if (rank == 0 && (src != r0 + r || src == slot))  // a row that stays is not rewritten
            reinterpret_cast<uint4*>((which ? vc : kc) + (row0 + r0 + r) * D)[cc] = val;
        }
        sep::fence_proxy_async_smem();  // later tensor copies refill these bytes
        __syncwarp();
        if (lane == 0) sep::mbar_arrive(&full[st]);  // plain stores, released by the arrive
      } else if (lane == 0) {
        // K/V rows are read once per step: evict them from L2 before the
        // metadata, q and outputs that the next launches need
        const uint64_t pol = sep::l2_evict_first_policy();
        sep::mbar_arrive_expect_tx(&full[st], SB);
#pragma unroll
        for (int j = 0; j < NB; ++j) {
          sep::tma_load_2d_hint(kt + j * kTileBytes, &map_k, 64 * j, static_cast<int32_t>(row0 + r0), &full[st], pol);
          sep::tma_load_2d_hint(vt + j * kTileBytes, &map_v, 64 * j, static_cast<int32_t>(row0 + r0), &full[st], pol);
        }
      }
      issued = ci + 1;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // before this warp's stores in the merge
  } else {
    // ---------------------------------------------------------- consumers
    const int kr = 16 * warp;  // this warp's rows of each chunk
    // Rotary table reads go before the grid-dependency wait: the table is
    // written by a launch that lets no later kernel start before it ends.
    // cq/ck: (cos, sin) pairs of the lane's dims f, f + 1 (index 2kk + h,
    // f = 16kk + 8h + 2tq) at the query's slot and at the lane's first row.
    float4 cq[ROPE ? DT : 1], ck[ROPE ? DT : 1];
    if constexpr (ROPE) {
      for (int e = threadIdx.x; e < D; e += 128) {
        const int t = e / (D / 2), i = e % (D / 2);
        const float2 cs = reinterpret_cast<const float2*>(p.rope)[(t ? 64 : 8) * (D / 2) + i];
        rope_c[t][i] = cs.x;
        rope_s[t][i] = cs.y;
      }
      const int mq = len > 0 ? len - 1 : 0;  // the query: the newest token's slot
      int r1 = rs + kr + gq;
      if (r1 > p.rope_rows - 1) r1 = p.rope_rows - 1;  // rows past len: never used
#pragma unroll
      for (int kk = 0; kk < DT / 2; ++kk)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int f = 16 * kk + 8 * h + 2 * tq;
          cq[2 * kk + h] = *reinterpret_cast<const float4*>(p.rope + static_cast<int64_t>(mq) * D + 2 * f);
          ck[2 * kk + h] = *reinterpret_cast<const float4*>(p.rope + static_cast<int64_t>(r1) * D + 2 * f);
        }
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");  // q, k_new, v_new
    uint32_t qb[DT][2];  // Q^T as the B operand: dims x heads (heads >= G are zero)
    {
      const T* qg = static_cast<const T*>(p.q) + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
#pragma unroll
      for (int kk = 0; kk < DT; ++kk) {
        const bool in = gq < G;
        qb[kk][0] = in ? *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * kk + 2 * tq) : 0u;
        qb[kk][1] = in ? *reinterpret_cast<const uint32_t*>(qg + gq * D + 16 * kk + 8 + 2 * tq) : 0u;
      }
    }
    // Positional-encoding shifting.  The lane's fragments hold dims f =
    // 16kk + 8h + 2tq + {0, 1} (kk < DT/2, h in {0, 1}: register h of the B
    // operand, registers 2h and 2h + 1 (rows gq, gq + 8) of the A operand),
    // and the partner dim f + D/2 sits in the same register of tile
    // kk + DT/2, so the rotation needs no data exchange.  ec/es[2kk + h]:
    // cos / sin at dims f, f + 1 of the lane's row rs + 64c + kr + gq of
    // chunk c, advanced chunk to chunk by the turn of 64 slots; row gq + 8
    // is one turn of 8 further.  The encoded scores use tf32 operands: a dot
    // product may take its terms in any order shared by both operands, so a
    // 16-dim tile is two k = 8 products, one over the lane's even dims
    // (2tq, 2tq + 8) and one over its odd dims, read straight from the bf16
    // fragments' registers.  qf[t][2h + e]: encoded q at dim 16t + 8h + 2tq + e.
    float2 ec[ROPE ? DT : 1], es[ROPE ? DT : 1];
    uint32_t qf[ROPE ? DT : 1][4];
    if constexpr (ROPE) {
      sep::named_bar_sync(1, 128);  // rope_c / rope_s are filled
#pragma unroll
      for (int kk = 0; kk < DT / 2; ++kk)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int i = 2 * kk + h;
          uint32_t lq[2], hq[2];
          rope_tf32(qb[kk][h], qb[kk + DT / 2][h], make_float2(cq[i].x, cq[i].z),
                    make_float2(cq[i].y, cq[i].w), lq, hq);
          qf[kk][2 * h] = lq[0];
          qf[kk][2 * h + 1] = lq[1];
          qf[kk + DT / 2][2 * h] = hq[0];
          qf[kk + DT / 2][2 * h + 1] = hq[1];
          ec[i] = make_float2(ck[i].x, ck[i].z);
          es[i] = make_float2(ck[i].y, ck[i].w);
        }
    }
    for (int ci = 0; ci < nchunks; ++ci) {
      const int c = chunk_of(ci);
      const int st = ci % kPipeStages;
      const int r0 = rs + c * ROWS;
      const int nr = re - r0 < ROWS ? re - r0 : ROWS;
      uint8_t* const kt = ring + st * SB;
      uint8_t* const vt = kt + NB * kTileBytes;
      if constexpr (ROPE) {
        if (c > 0) {  // (chunks in ascending order)
#pragma unroll
          for (int i = 0; i < DT; ++i) {
            const int f = 16 * (i / 2) + 8 * (i & 1) + 2 * tq;
            cturn(ec[i], es[i], *reinterpret_cast<const float2*>(&rope_c[1][f]),
                  *reinterpret_cast<const float2*>(&rope_s[1][f]));
          }
        }
      }
      if (!__all_sync(0xffffffffu, sep::mbar_wait(&full[st], (ci / kPipeStages) & 1, &abort_flag, p.err)))
        break;
      if (kr < nr) {
        bool wrote = false;
        if (FUSED && !flush && slot >= r0 + kr && slot < r0 + kr + 16 && slot < r0 + nr) {
          // the new token (the last row without a flush): from k_new/v_new,
          // also stored into the cache
          const int r = slot - r0;
          const uint4* kn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.k_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
          const uint4* vn = reinterpret_cast<const uint4*>(static_cast<const T*>(p.v_new) + (static_cast<int64_t>(b) * p.Hkv + g) * D);
          for (int e = lane; e < 2 * CH; e += 32) {
            const int which = e / CH, cc = e % CH;
            const uint4 val = (which ? vn : kn)[cc];
            *reinterpret_cast<uint4*>((which ? vt : kt) + swz(r, 8 * cc)) = val;
            reinterpret_cast<uint4*>((which ? vc : kc) + (row0 + r0 + r) * D)[cc] = val;
          }
          wrote = true;
        }
        // V rows of this warp past the chunk's end (whatever the copy
        // brought in): P is 0 there, and 0 * garbage may be NaN
        const int vr = nr - kr < 16 ? nr - kr : 16;
        for (int e = lane; e < (16 - vr) * CH; e += 32)
          *reinterpret_cast<uint4*>(vt + swz(kr + vr + e / CH, 8 * (e % CH))) = make_uint4(0, 0, 0, 0);
        if (wrote || vr < 16) sep::fence_proxy_async_smem();  // refilled by tensor copies later
        __syncwarp();
        // all K and V fragments of the warp's 16 rows first: each ldmatrix
        // waits ~100 cycles, back to back they overlap
        const uint32_t kb = sep::smem_u32(kt), vb = sep::smem_u32(vt);
        uint32_t ka[DT][4], va[DT][4];
#pragma unroll
        for (int kk = 0; kk < DT; ++kk)
          ldsm_x4(kb + swz(kr + (lane & 7) + ((lane >> 3) & 1) * 8, 16 * kk + (lane >> 4) * 8), ka[kk]);
#pragma unroll
        for (int dt = 0; dt < DT; ++dt)
          ldsm_x4_t(vb + swz(kr + (lane & 7) + (lane >> 4) * 8, 16 * dt + ((lane >> 3) & 1) * 8), va[dt]);
        // S^T = K Q^T for the warp's 16 keys (rows) x 8 heads, four chains
        float sacc[4][4] = {};
        if constexpr (ROPE) {
#pragma unroll
          for (int kk = 0; kk < DT / 2; ++kk) {
            // encoded K of tile kk (kl) and of its partner tile kk + DT/2
            // (kh): [register of the bf16 fragment][even / odd dim]
            uint32_t kl[4][2], kh[4][2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int f = 16 * kk + 8 * h + 2 * tq, i = 2 * kk + h;
              rope_tf32(ka[kk][2 * h], ka[kk + DT / 2][2 * h], ec[i], es[i], kl[2 * h], kh[2 * h]);
              float2 c8 = ec[i], s8 = es[i];
              cturn(c8, s8, *reinterpret_cast<const float2*>(&rope_c[0][f]),
                    *reinterpret_cast<const float2*>(&rope_s[0][f]));
              rope_tf32(ka[kk][2 * h + 1], ka[kk + DT / 2][2 * h + 1], c8, s8, kl[2 * h + 1],
                        kh[2 * h + 1]);
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              mma1688(sacc[e], kl[0][e], kl[1][e], kl[2][e], kl[3][e], qf[kk][e], qf[kk][2 + e]);
              mma1688(sacc[2 + e], kh[0][e], kh[1][e], kh[2][e], kh[3][e], qf[kk + DT / 2][e],
                      qf[kk + DT / 2][2 + e]);
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < DT; ++kk) mma16816(sacc[kk & 3], ka[kk], qb[kk][0], qb[kk][1]);
        }
        // x0/x1: key kr + gq, heads 2tq / 2tq + 1; x2/x3: key kr + gq + 8
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          x[e] = ((sacc[0][e] + sacc[1][e]) + (sacc[2][e] + sacc[3][e])) * p.scale_log2;
        if (kr + gq >= nr) x[0] = x[1] = -INFINITY;
        if (kr + gq + 8 >= nr) x[2] = x[3] = -INFINITY;
        // the reference maxima move only when a score exceeds them by more
        // than 2^8 (always on the warp's first keys); otherwise P <= 256
        const bool up = x[0] > m0 + kLazyLog2 || x[2] > m0 + kLazyLog2 ||
                        x[1] > m1 + kLazyLog2 || x[3] > m1 + kLazyLog2;
        if (__any_sync(0xffffffffu, up)) {
          float c0 = fmaxf(x[0], x[2]), c1 = fmaxf(x[1], x[3]);  // column maxima
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            c0 = fmaxf(c0, __shfl_xor_sync(0xffffffffu, c0, off));
            c1 = fmaxf(c1, __shfl_xor_sync(0xffffffffu, c1, off));
          }
          const float n0 = fmaxf(m0, c0), n1 = fmaxf(m1, c1);
          const float al0 = exp2f(m0 - n0), al1 = exp2f(m1 - n1);  // 0 on the first keys
          l0 *= al0;
          l1 *= al1;
#pragma unroll
          for (int dt = 0; dt < DT; ++dt) {
            o[dt][0] *= al0;
            o[dt][1] *= al1;
            o[dt][2] *= al0;
            o[dt][3] *= al1;
          }
          m0 = n0;
          m1 = n1;
        }
        const float p0 = exp2f(x[0] - m0), p1 = exp2f(x[1] - m1);
        const float p2 = exp2f(x[2] - m0), p3 = exp2f(x[3] - m1);
        l0 += p0 + p2;
        l1 += p1 + p3;
        // P^T (keys x heads) as the B operand: transpose the 8x8 blocks
        const uint32_t pb0 = movmatrix_t(sep::pack_bf16x2(p0, p1));
        const uint32_t pb1 = movmatrix_t(sep::pack_bf16x2(p2, p3));
        // O^T += V^T P^T, V^T as the A operand (ldmatrix.trans of V rows)
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) mma16816(o[dt], va[dt], pb0, pb1);
      }
      __syncwarp();
      if (lane == 0) sep::mbar_arrive(&empty[st]);
    }
    // this lane's sums -> the column sums of heads 2tq, 2tq + 1
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
  }
  __syncthreads();
  if (abort_flag) {
    // a wait gave up: let this CTA's copies land before it can exit
    if (threadIdx.x == 4 * 32) {
      int dummy = 0;
      for (int c = issued - kPipeStages < 0 ? 0 : issued - kPipeStages; c < issued; ++c)
        sep::mbar_wait(&full[c % kPipeStages], (c / kPipeStages) & 1, &dummy, nullptr);
    }
    __syncthreads();
  }
  sep::cluster_wait();
  if (warp < 4) {
    // send this warp's partial: dims of slice t go to CTA t
    const uint32_t recv_s = sep::smem_u32(recv_o) + (rank * 4 + warp) * PART * 4;
    const uint32_t rm_s = sep::smem_u32(&rm[rank][warp][0]), rl_s = sep::smem_u32(&rl[rank][warp][0]);
    const int h0 = 2 * tq;
    if (h0 < G) {
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int d = 16 * dt + gq + 8 * r;
          const int t = d / DQ;
          const uint32_t dst = sep::cluster_addr_of(recv_s + ((d - t * DQ) * G + h0) * 4, t);
          const uint32_t bar = sep::cluster_addr(&mrg, t);
          if (G >= 2)
            sep::st_async_v2f32(dst, o[dt][2 * r], o[dt][2 * r + 1], bar);
          else
            sep::st_async_f32(dst, o[dt][2 * r], bar);
        }
      }
      if (gq == 0) {
#pragma unroll
        for (int t = 0; t < NCL; ++t) {
          const uint32_t bar = sep::cluster_addr(&mrg, t);
          sep::st_async_f32(sep::cluster_addr_of(rm_s + h0 * 4, t), m0, bar);
          sep::st_async_f32(sep::cluster_addr_of(rl_s + h0 * 4, t), l0, bar);
          if (h0 + 1 < G) {
            sep::st_async_f32(sep::cluster_addr_of(rm_s + (h0 + 1) * 4, t), m1, bar);
            sep::st_async_f32(sep::cluster_addr_of(rl_s + (h0 + 1) * 4, t), l1, bar);
          }
        }
      }
    }
  }
  sep::mbar_wait_cluster(&mrg, 0, p.err);
  // merge the NCL x 4 partials of this CTA's DQ x G outputs, one element of
  // the [d][head] layout per thread (consecutive words)
  T* const out = static_cast<T*>(p.out);
  for (int f = threadIdx.x; f < PART; f += kPipeThreads) {
    const int h = f % G, d = rank * DQ + f / G;
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < NCL * 4; ++k) M = fmaxf(M, rm[k / 4][k % 4][h]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int k = 0; k < NCL * 4; ++k) {
      const float mk = rm[k / 4][k % 4][h];
      const float wgt = mk == -INFINITY ? 0.f : exp2f(mk - M);
      L += rl[k / 4][k % 4][h] * wgt;
      acc += recv_o[k * PART + f] * wgt;
    }
    out[(static_cast<int64_t>(b) * p.Hq + g * G + h) * D + d] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
    if (p.lse && d == 0)
      p.lse[static_cast<int64_t>(b) * p.Hq + g * G + h] =
          L > 0.f ? (M + log2f(L)) * 0.69314718055994530942f : -INFINITY;
  }
  if constexpr (FUSED) {
    if (flush && rank > 0 && rs < re) {
      // The merge has received the first CTA's partials, sent after it had
      // loaded every one of its rows: its sources are all read, so this
      // CTA's rows can now move in place (staged through ring stage 0).
      __syncthreads();
      compact_in_place<T, D>(p, b, g, rs, re, slot, ROWS, kPipeThreads, reinterpret_cast<T*>(ring),
                             reinterpret_cast<T*>(ring + ROWS * D * 2));
    }
  }
}

// Maximum dynamic shared memory for `kern` on the current device, set once.
template <typename K>
bool allow_smem(K kern, int smem, bool* done) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem <= 48 * 1024 || dev < 0 || dev >= 64 || done[dev]) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return false;
  done[dev] = true;
  return true;
}

template <typename T, int D, int G, bool FUSED, bool CLUSTER>
int launch_one(const DecodeParams& p, cudaStream_t st) {
  constexpr bool TC = sizeof(T) == 2;  // bf16: streamed tensor-core kernel; fp32: exact FMA kernel
  constexpr int smem = TC ? pipe_smem_bytes<D, G>() : 2 * ROWS * D * static_cast<int>(sizeof(T));
  const int ncl = TC ? kPipeCluster : (CLUSTER ? kMaxClusterSplits : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(TC ? kPipeCluster : (CLUSTER ? kMaxClusterSplits : p.nsplit), p.Hkv, p.B);
  cfg.blockDim = dim3(TC ? kPipeThreads : kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na].val.programmaticStreamSerializationAllowed = 1;
  ++na;
  if (ncl > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = ncl;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  static bool attr_set[64] = {false};
  if constexpr (TC) {
    CUtensorMap mk, mv;
    static bool attr_rope[64] = {false}, attr_gen[64] = {false};
    auto kern = p.rope ? k_decode_pipe<D, G, FUSED, true, false> : k_decode_pipe<D, G, FUSED, false, false>;
    bool* done = p.rope ? attr_rope : attr_set;
    if constexpr (!FUSED) {
      if (p.prefix) {  // rows gathered by index: the tensor maps stay unused
        memset(&mk, 0, sizeof mk);
        memset(&mv, 0, sizeof mv);
        kern = k_decode_pipe<D, G, false, false, true>;
        done = attr_gen;
      }
    }
    if (!p.prefix) {
      // the K and V arrays as [layers * B * Hkv * cap, D] rows
      const int64_t rows = static_cast<int64_t>(p.layers) * p.B * p.Hkv * p.cap;
      if (rows > 0x7fffffffLL) return SEP_ETOOBIG;
      if (!sep::make_rows_map(&mk, p.kc, rows, D, ROWS) || !sep::make_rows_map(&mv, p.vc, rows, D, ROWS))
        return SEP_ECUDA;
    }
    if (!allow_smem(kern, smem, done)) return SEP_ECUDA;
    if (cudaLaunchKernelEx(&cfg, kern, p, mk, mv) != cudaSuccess) return SEP_ECUDA;
  } else {
    auto kern = k_decode<T, D, G, FUSED, CLUSTER>;
    if (!allow_smem(kern, smem, attr_set)) return SEP_ECUDA;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return SEP_ECUDA;
  }
  return sep::launch_status();
}

template <typename T, int D, bool FUSED = false>
int launch_g(const DecodeParams& p, int G, cudaStream_t st) {
  const bool cl = p.nsplit <= kMaxClusterSplits;
  switch (G) {
    case 1: return cl ? launch_one<T, D, 1, FUSED, true>(p, st) : launch_one<T, D, 1, FUSED, false>(p, st);
    case 2: return cl ? launch_one<T, D, 2, FUSED, true>(p, st) : launch_one<T, D, 2, FUSED, false>(p, st);
    case 4: return cl ? launch_one<T, D, 4, FUSED, true>(p, st) : launch_one<T, D, 4, FUSED, false>(p, st);
    case 8: return cl ? launch_one<T, D, 8, FUSED, true>(p, st) : launch_one<T, D, 8, FUSED, false>(p, st);
    default: return SEP_EINVAL;
  }
}

bool cache_ok(const sepcache* c) { return sep::cache_valid(c); }

struct WsLayout {
  size_t ml, o, ticket;
};
WsLayout ws_layout_of(int B, int Hq, int Hkv, int rows, int D) {
  const size_t nsplit = (rows + ROWS - 1) / ROWS;
  WsLayout w;
  w.ml = (static_cast<size_t>(B) * Hq * nsplit * 2 * 4 + 255) / 256 * 256;
  w.o = (static_cast<size_t>(B) * Hq * nsplit * D * 4 + 255) / 256 * 256;
  w.ticket = (static_cast<size_t>(B) * Hkv * 4 + 255) / 256 * 256;
  return w;
}
WsLayout ws_layout(const sepcache* c, int Hq) { return ws_layout_of(c->B, Hq, c->Hkv, c->cap, c->D); }

}  // namespace

extern "C" size_t sep_attn_decode_workspace(const sepcache* c, int Hq) {
  if (!cache_ok(c) || Hq < 1) return 0;
  const WsLayout w = ws_layout(c, Hq);
  return w.ml + w.o + w.ticket;
}

extern "C" int sep_attn_decode(const sepcache* c, int layer, const void* q, int Hq, float scale,
                               void* out, float* lse, void* workspace, size_t workspace_bytes,
                               void* stream) {
  if (!c) return SEP_ENULL;
  if (!cache_ok(c)) return SEP_EINVAL;
  if (layer < 0 || layer >= c->layers) return SEP_EINVAL;
  if (Hq < 1 || Hq % c->Hkv != 0) return SEP_EINVAL;
  const int G = Hq / c->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SEP_EINVAL;
  if (!q || !out || !workspace) return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(out) || !sep::aligned16(workspace)) return SEP_EALIGN;
  const WsLayout w = ws_layout(c, Hq);
  if (workspace_bytes < w.ml + w.o + w.ticket) return SEP_EINVAL;
  DecodeParams p = {};
  p.q = q;
  p.kc = c->k;
  p.vc = c->v;
  p.counts = c->counts;
  p.plan = c->plan;
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.layers = c->layers;
  p.out = out;
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.part_ml = reinterpret_cast<float*>(ws);
  p.part_o = reinterpret_cast<float*>(ws + w.ml);
  p.ticket = reinterpret_cast<int32_t*>(ws + w.ml + w.o);
  p.err = sep::device_error_word();
  p.layer = layer;
  p.B = c->B;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.cap = c->cap;
  p.nsplit = (c->cap + ROWS - 1) / ROWS;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(c->D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  p.rope = c->rope_theta > 0.f ? c->rope : nullptr;
  p.rope_rows = c->rope_rows;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->dtype == SEP_BF16)
    return c->D == 64 ? launch_g<__nv_bfloat16, 64>(p, G, st) : launch_g<__nv_bfloat16, 128>(p, G, st);
  return c->D == 64 ? launch_g<float, 64>(p, G, st) : launch_g<float, 128>(p, G, st);
}

extern "C" int sep_attn_decode_step(const sepcache* c, int layer, const void* q,
                                    const void* k_new, const void* v_new,
                                    const uint8_t* is_sep_new, int Hq, float scale, void* out,
                                    float* lse, void* workspace, size_t workspace_bytes,
                                    void* stream) {
  if (!c) return SEP_ENULL;
  if (!cache_ok(c)) return SEP_EINVAL;
  if (layer < 0 || layer >= c->layers) return SEP_EINVAL;
  if (Hq < 1 || Hq % c->Hkv != 0) return SEP_EINVAL;
  const int G = Hq / c->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SEP_EINVAL;
  if (!q || !out || !workspace || !k_new || !v_new || (layer == 0 && !is_sep_new)) return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(out) || !sep::aligned16(workspace) ||
      !sep::aligned16(k_new) || !sep::aligned16(v_new))
    return SEP_EALIGN;
  const WsLayout w = ws_layout(c, Hq);
  if (workspace_bytes < w.ml + w.o + w.ticket) return SEP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (layer == 0) {
    const int rc = sep::cache_advance(c, is_sep_new, st);
    if (rc != SEP_OK) return rc;
  }
  DecodeParams p = {};
  p.q = q;
  p.kc = c->k;
  p.vc = c->v;
  p.counts = c->counts;
  p.plan = c->plan;
  p.k_new = k_new;
  p.v_new = v_new;
  p.layers = c->layers;
  p.out = out;
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.part_ml = reinterpret_cast<float*>(ws);
  p.part_o = reinterpret_cast<float*>(ws + w.ml);
  p.ticket = reinterpret_cast<int32_t*>(ws + w.ml + w.o);
  p.err = sep::device_error_word();
  p.layer = layer;
  p.B = c->B;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.cap = c->cap;
  p.nsplit = (c->cap + ROWS - 1) / ROWS;
  p.early = layer > 0;  // the step's metadata was advanced in the layer-0 call
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(c->D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  p.rope = c->rope_theta > 0.f ? c->rope : nullptr;
  p.rope_rows = c->rope_rows;
  if (c->dtype == SEP_BF16)
    return c->D == 64 ? launch_g<__nv_bfloat16, 64, true>(p, G, st)
                      : launch_g<__nv_bfloat16, 128, true>(p, G, st);
  return c->D == 64 ? launch_g<float, 64, true>(p, G, st) : launch_g<float, 128, true>(p, G, st);
}

// ---------------------------------------------------------------------------
// Decode for callers that cannot allocate device memory.
//
// Some callers cannot hand this library a workspace: a plug-in that a host
// framework calls with only the tensors of the call (the framework owns
// every device allocation), or a serving loop whose device memory is fully
// reserved for its KV pool, where a new cudaMalloc would fail or stall the
// device.  This entry point keeps the split-K partials and tickets in a
// fixed scratch array inside the library instead.  Every GPU that loads the
// library holds the array (about 4.1 MiB) until the process exits; every
// call shares it, so calls that overlap on the GPU race on it.
//
// Only one kernel form reads or writes the array: the exact fp32 decode of a
// cache with more than kMaxClusterSplits splits of 64 rows, whose splits
// merge through memory with an atomic ticket.  The bf16 kernel and the fp32
// kernel with at most kMaxClusterSplits splits merge inside a thread-block
// cluster and never touch it, so the size limits and the ticket clear apply
// to the first form only.
namespace {

constexpr int kNoAllocMaxPartials = 8192;  // B * Hq * splits, splits = ceil(cap / 64)
constexpr int kNoAllocMaxTickets = 4096;   // B * Hkv
constexpr size_t kNoAllocMlBytes = static_cast<size_t>(kNoAllocMaxPartials) * 2 * 4;
constexpr size_t kNoAllocOBytes = static_cast<size_t>(kNoAllocMaxPartials) * 128 * 4;
constexpr size_t kNoAllocTicketBytes = static_cast<size_t>(kNoAllocMaxTickets) * 4;
constexpr size_t kNoAllocBytes = kNoAllocMlBytes + kNoAllocOBytes + kNoAllocTicketBytes;
constexpr int kNoAllocMaxDevices = 64;

}  // namespace

// The scratch itself.  In host code this name is only a stand-in for the
// array, not its device address: the address is looked up per device.
static __device__ __align__(256) uint8_t g_decode_scratch[kNoAllocBytes];

namespace {

// Device address of the scratch array, per device.  Set once per device
// (the first call on it, with that device current); a race between two
// host threads making that first call stores the same value twice, and the
// atomic makes that well defined.  The address is not refreshed after
// cudaDeviceReset: a process that resets a device must not use this entry
// point on it afterwards.
std::atomic<uint8_t*> g_decode_scratch_addr[kNoAllocMaxDevices];

}  // namespace

extern "C" int sep_attn_decode_noalloc(const sepcache* c, int layer, const void* q, int Hq,
                                       float scale, void* out, float* lse, void* stream) {
  if (!c) return SEP_ENULL;
  if (!cache_ok(c)) return SEP_EINVAL;
  if (layer < 0 || layer >= c->layers) return SEP_EINVAL;
  if (Hq < 1 || Hq % c->Hkv != 0) return SEP_EINVAL;
  const int G = Hq / c->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SEP_EINVAL;
  if (!q || !out) return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(out)) return SEP_EALIGN;
  const int nsplit = (c->cap + ROWS - 1) / ROWS;
  // the only kernel form that merges through the scratch array
  const bool uses_scratch = c->dtype == SEP_F32 && nsplit > kMaxClusterSplits;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DecodeParams p = {};
  if (uses_scratch) {
    if (static_cast<int64_t>(c->B) * Hq * nsplit > kNoAllocMaxPartials ||
        static_cast<int64_t>(c->B) * c->Hkv > kNoAllocMaxTickets)
      return SEP_ETOOBIG;
    // set-up, once per device with that device current: the device address
    // of the scratch array (the host-side symbol is not a device address)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
      return SEP_ECUDA;
    uint8_t* scratch = g_decode_scratch_addr[dev].load(std::memory_order_acquire);
    if (!scratch) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return SEP_ECUDA;
      scratch = static_cast<uint8_t*>(ptr);
      g_decode_scratch_addr[dev].store(scratch, std::memory_order_release);
    }
    int32_t* tickets = reinterpret_cast<int32_t*>(scratch + kNoAllocMlBytes + kNoAllocOBytes);
    // the tickets must start at zero (the array keeps the previous call's contents)
    if (cudaMemsetAsync(tickets, 0, static_cast<size_t>(c->B) * c->Hkv * 4, st) != cudaSuccess)
      return SEP_ECUDA;
    p.part_ml = reinterpret_cast<float*>(scratch);
    p.part_o = reinterpret_cast<float*>(scratch + kNoAllocMlBytes);
    p.ticket = tickets;
  }
  p.q = q;
  p.kc = c->k;
  p.vc = c->v;
  p.counts = c->counts;
  p.plan = c->plan;
  p.k_new = nullptr;
  p.v_new = nullptr;
  p.layers = c->layers;
  p.out = out;
  p.lse = lse;
  p.err = sep::device_error_word();
  p.layer = layer;
  p.B = c->B;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.cap = c->cap;
  p.nsplit = nsplit;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(c->D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  p.rope = c->rope_theta > 0.f ? c->rope : nullptr;
  p.rope_rows = c->rope_rows;
  if (c->dtype == SEP_BF16)
    return c->D == 64 ? launch_g<__nv_bfloat16, 64>(p, G, st) : launch_g<__nv_bfloat16, 128>(p, G, st);
  return c->D == 64 ? launch_g<float, 64>(p, G, st) : launch_g<float, 128>(p, G, st);
}

// ---------------------------------------------------------------------------
// Mask-based generation: the newest token attends over the full history with
// the Sep-Attention kept set of its row (the study's generate mask: the
// prefill mask's rule for a query of length 1), no rows evicted.
namespace {
bool gen_args_ok(int B, int Hq, int Hkv, int S, int T, int D, int a, int n, int dtype) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || B > 65535 || Hkv > 65535) return false;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return false;
  if (S < 1 || T < 1 || T > S || a < 0 || n < 1) return false;
  if (static_cast<int64_t>(B) * Hkv * S >= (1LL << 31)) return false;
  (void)D;
  (void)dtype;
  return true;
}
}  // namespace

extern "C" size_t sep_attn_decode_masked_workspace(int B, int Hq, int Hkv, int S, int D) {
  if (!gen_args_ok(B, Hq, Hkv, S, S, D, 0, 1, SEP_BF16) || (D != 64 && D != 128)) return 0;
  const WsLayout w = ws_layout_of(B, Hq, Hkv, S, D);
  return w.ml + w.o + w.ticket;
}

extern "C" int sep_attn_decode_masked(const void* q, const void* k, const void* v, int dtype,
                                      const int32_t* prefix, const int32_t* idx, int B, int Hq,
                                      int Hkv, int S, int T, int D, int a, int n, float scale,
                                      void* out, float* lse, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (dtype != SEP_F32 && dtype != SEP_BF16) return SEP_EDTYPE;
  if (D != 64 && D != 128) return SEP_EDTYPE;
  if (!gen_args_ok(B, Hq, Hkv, S, T, D, a, n, dtype)) return SEP_EINVAL;
  if (!q || !k || !v || !prefix || !idx || !out) return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(k) || !sep::aligned16(v) || !sep::aligned16(out))
    return SEP_EALIGN;
  const WsLayout w = ws_layout_of(B, Hq, Hkv, T, D);
  if (dtype == SEP_F32) {  // the exact kernel merges splits through the workspace
    if (!workspace) return SEP_ENULL;
    if (!sep::aligned16(workspace)) return SEP_EALIGN;
    if (workspace_bytes < w.ml + w.o + w.ticket) return SEP_EINVAL;
  }
  DecodeParams p = {};
  p.q = q;
  p.kc = k;
  p.vc = v;
  p.out = out;
  p.lse = lse;
  if (workspace) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    p.part_ml = reinterpret_cast<float*>(ws);
    p.part_o = reinterpret_cast<float*>(ws + w.ml);
    p.ticket = reinterpret_cast<int32_t*>(ws + w.ml + w.o);
  }
  p.err = sep::device_error_word();
  p.layer = 0;
  p.layers = 1;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.cap = T;  // at most T kept rows
  p.nsplit = (T + ROWS - 1) / ROWS;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  p.prefix = prefix;
  p.idx = idx;
  p.S = S;
  p.T = T;
  p.a = a;
  p.n = n;
  const int G = Hq / Hkv;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SEP_BF16)
    return D == 64 ? launch_g<__nv_bfloat16, 64>(p, G, st) : launch_g<__nv_bfloat16, 128>(p, G, st);
  return D == 64 ? launch_g<float, 64>(p, G, st) : launch_g<float, 128>(p, G, st);
}
