// Separator flags, per-sequence separator index lists, and kept-pair counts.
//
// The separator set and the kept rule follow the "HKUDS047: SepLLM ..." study,
// sections "Separator Tokens" and "SepAttention" (token_id in
// separator_token_ids; initial + separator + local-window columns AND the
// causal mask).  The index list is the prefix-scan compaction of the flags
// that lets the attention kernel fetch separator rows by position.
#include <string.h>

#include "common.cuh"

namespace {

constexpr int kMaxSepIds = 32;
struct SepIdSet {
  int32_t id[kMaxSepIds];
  int n;
};

__global__ void k_flags_from_ids(const int32_t* __restrict__ ids, int64_t n_tok, SepIdSet set,
                                 uint8_t* __restrict__ is_sep) {
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the ids' producer
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (; t < n_tok; t += stride) {
    int32_t v = ids[t];
    uint8_t f = 0;
#pragma unroll 4
    for (int k = 0; k < set.n; ++k) f |= (v == set.id[k]);
    is_sep[t] = f;
  }
}

// One CTA per (chunk of positions, sequence); a chunk is kPer positions per
// thread, and a CTA has as many warps as its chunk needs (at most 32).  Warp
// w of the CTA owns kPer x 32 consecutive positions, lane l the positions
// 32e + l (e < kPer), so that flag reads and prefix writes are coalesced.  A
// warp ranks its separators with ballots, one block-wide scan of the warp
// totals gives the offsets.  With several chunks per sequence each CTA first
// counts the separators before its chunk and in the whole sequence (read
// from L2); no CTA waits on another.  FROM_IDS: the flags are computed from
// the token ids here (and written out), so one launch replaces the flag
// kernel and this one.
constexpr int kScanThreads = 1024;
constexpr int kPer = 16;
constexpr int kChunkMax = kScanThreads * kPer;

__device__ __forceinline__ int block_sum(int v, int* red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  int s = 0;
  if (w == 0) {
    s = l < nw ? red[l] : 0;
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (l == 0) red[32] = s;
  }
  __syncthreads();
  return red[32];
}

// Membership in the id set: the host pads id[n..32) with id[0], so all 32
// fixed slots are compared (fixed indices keep the set in the parameter bank).
__device__ __forceinline__ bool in_set(int32_t v, const SepIdSet& set) {
  bool f = false;
#pragma unroll
  for (int k = 0; k < kMaxSepIds; ++k) f |= (v == set.id[k]);
  return f;
}

template <bool FROM_IDS>
__global__ void __launch_bounds__(kScanThreads) k_build_index(
    const uint8_t* __restrict__ is_sep, const int32_t* __restrict__ ids, const SepIdSet set,
    uint8_t* __restrict__ is_sep_out, int S, int32_t* __restrict__ prefix,
    int32_t* __restrict__ idx, int32_t* __restrict__ count) {
  __shared__ int red[33];
  __shared__ int wsum[33];
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the flags' (or ids') producer
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int b = blockIdx.y;
  const int chunk0 = static_cast<int>(blockIdx.x * blockDim.x) * kPer;  // < S < 2^31
  const uint8_t* f = is_sep + static_cast<int64_t>(b) * S;
  const int32_t* tok = ids + static_cast<int64_t>(b) * S;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  auto flag_at = [&](int p) -> bool { return FROM_IDS ? in_set(tok[p], set) : f[p] != 0; };

  // separators before the chunk, and in the whole sequence (every chunk's
  // CTA counts the whole sequence; with flags in 16-byte-aligned rows, 16
  // flags per load: a byte's top bit is set where the byte is nonzero, and
  // the four 0/1 bytes of a word are summed by a multiply)
  int before = 0, total = -1;
  if (gridDim.x > 1) {
    int tot = 0;
    if (!FROM_IDS && (reinterpret_cast<uintptr_t>(f) & 15u) == 0) {
      const uint4* f4 = reinterpret_cast<const uint4*>(f);
      const int n16 = S >> 4;  // chunk0 is a multiple of 16
      for (int q = threadIdx.x; q < n16; q += blockDim.x) {
        const uint4 w = f4[q];
        auto nz4 = [](uint32_t x) {  // nonzero bytes of x
          const uint32_t hi = (((x & 0x7f7f7f7fu) + 0x7f7f7f7fu) | x) & 0x80808080u;
          return static_cast<int>(((hi >> 7) * 0x01010101u) >> 24);
        };
        const int v = nz4(w.x) + nz4(w.y) + nz4(w.z) + nz4(w.w);
        tot += v;
        before += (16 * q < chunk0) ? v : 0;
      }
      for (int p = (n16 << 4) + threadIdx.x; p < S; p += blockDim.x) {
        const int v = f[p] != 0;
        tot += v;
        before += (p < chunk0) ? v : 0;
      }
    } else {
      for (int p = threadIdx.x; p < S; p += blockDim.x) {
        const int v = flag_at(p);
        tot += v;
        before += (p < chunk0) ? v : 0;
      }
    }
    before = block_sum(before, red);
    total = block_sum(tot, red);
  }

  // this warp's flags: bit e of `bits` is position w0 + 32e + lane
  const int w0 = chunk0 + warp * 32 * kPer;
  uint32_t bits = 0;
  int wtot = 0;
  if (FROM_IDS) {
    // all loads first: a flag store between them would keep the compiler
    // from having the kPer loads in flight together
    int32_t tv[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int pos = w0 + 32 * e + lane;
      tv[e] = pos < S ? tok[pos] : 0;
    }
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int pos = w0 + 32 * e + lane;
      const bool fl = pos < S && in_set(tv[e], set);
      if (pos < S) is_sep_out[static_cast<int64_t>(b) * S + pos] = fl ? 1 : 0;
      bits |= static_cast<uint32_t>(fl) << e;
    }
  } else {
#pragma unroll
    for (int e = 0; e < kPer; ++e) {
      const int pos = w0 + 32 * e + lane;
      bits |= static_cast<uint32_t>(pos < S && f[pos] != 0) << e;
    }
  }
#pragma unroll
  for (int e = 0; e < kPer; ++e) wtot += __popc(__ballot_sync(0xffffffffu, (bits >> e) & 1u));
  // exclusive scan of the warp totals
  if (lane == 0) wsum[warp] = wtot;
  __syncthreads();
  if (warp == 0) {
    const int x = lane < nwarps ? wsum[lane] : 0;
    int xi = x;
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, xi, o);
      if (lane >= o) xi += y;
    }
    wsum[lane] = xi - x;
    if (lane == 31) wsum[32] = xi;  // the chunk's total
  }
  __syncthreads();
  if (total < 0) total = wsum[32];  // one chunk: the sequence's total

  int32_t* pre = prefix + static_cast<int64_t>(b) * (S + 1);
  int32_t* ix = idx + static_cast<int64_t>(b) * S;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    pre[0] = 0;
    count[b] = total;
  }
  int run = before + wsum[warp];
#pragma unroll
  for (int e = 0; e < kPer; ++e) {
    const int pos = w0 + 32 * e + lane;
    const uint32_t bal = __ballot_sync(0xffffffffu, (bits >> e) & 1u);
    const int rank = run + __popc(bal & lt);
    if (pos < S) {
      const bool fl = (bits >> e) & 1u;
      if (fl) ix[rank] = static_cast<int32_t>(pos);
      pre[pos + 1] = rank + static_cast<int>(fl);
      // idx slots at or after the total count are padding
      if (pos >= total) ix[pos] = -1;
    }
    run += __popc(bal);
  }
}

// Threads of a scan CTA: one chunk of S when it fits, whole warps.
int scan_threads(int S) {
  if (S > kChunkMax) return kScanThreads;
  const int warps = (S + 32 * kPer - 1) / (32 * kPer);
  return warps * 32;
}

// Closed form of one row's kept count: window [lo, i] + initial tokens left
// of it + separators in [a, lo), lo = max(0, i - n + 1).
__global__ void k_count_pairs(const int32_t* __restrict__ prefix, int S, int a, int n,
                              int64_t* __restrict__ kept) {
  __shared__ long long red[32];
  const int b = blockIdx.x;
  const int32_t* pre = prefix + static_cast<int64_t>(b) * (S + 1);
  const int aa = a < S ? a : S;
  long long acc = 0;
  for (int i = threadIdx.x; i < S; i += blockDim.x) {
    int lo = i - n + 1;
    if (lo < 0) lo = 0;
    long long c = static_cast<long long>(i - lo + 1) + (a < lo ? a : lo);
    if (lo > aa) c += pre[lo] - pre[aa];
    acc += c;
  }
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    long long s = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0;
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) kept[b] = s;
  }
}

}  // namespace

extern "C" int sep_flags_from_ids(const int32_t* ids, int64_t n_tok, const int32_t* sep_ids,
                                  int n_sep_ids, uint8_t* is_sep, void* stream) {
  if (n_tok < 0 || n_sep_ids < 1 || n_sep_ids > kMaxSepIds) return SEP_EINVAL;
  if (!sep_ids) return SEP_ENULL;
  if (n_tok == 0) return SEP_OK;
  if (!ids || !is_sep) return SEP_ENULL;
  SepIdSet set;
  memset(&set, 0, sizeof set);
  set.n = n_sep_ids;
  for (int k = 0; k < n_sep_ids; ++k) set.id[k] = sep_ids[k];
  int64_t blocks = (n_tok + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (sep::launch_pdl(k_flags_from_ids, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                      static_cast<cudaStream_t>(stream), ids, n_tok, set, is_sep) != cudaSuccess)
    return SEP_ECUDA;
  return sep::launch_status();
}

extern "C" int sep_build_index(const uint8_t* is_sep, int B, int S, int32_t* prefix, int32_t* idx,
                               int32_t* count, void* stream) {
  if (B < 1 || S < 1 || B > 65535) return SEP_EINVAL;
  if (!is_sep || !prefix || !idx || !count) return SEP_ENULL;
  const int threads = scan_threads(S);
  const int chunk = threads * kPer;
  SepIdSet none;
  memset(&none, 0, sizeof none);
  dim3 grid((S + chunk - 1) / chunk, B);
  if (sep::launch_pdl(k_build_index<false>, grid, dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), is_sep, static_cast<const int32_t*>(nullptr),
                      none, static_cast<uint8_t*>(nullptr), S, prefix, idx, count) != cudaSuccess)
    return SEP_ECUDA;
  return sep::launch_status();
}

extern "C" int sep_build_index_from_ids(const int32_t* ids, int B, int S, const int32_t* sep_ids,
                                        int n_sep_ids, uint8_t* is_sep, int32_t* prefix,
                                        int32_t* idx, int32_t* count, void* stream) {
  if (B < 1 || S < 1 || B > 65535 || n_sep_ids < 1 || n_sep_ids > kMaxSepIds) return SEP_EINVAL;
  if (!sep_ids) return SEP_ENULL;
  if (!ids || !is_sep || !prefix || !idx || !count) return SEP_ENULL;
  SepIdSet set;
  memset(&set, 0, sizeof set);
  set.n = n_sep_ids;
  for (int k = 0; k < kMaxSepIds; ++k) set.id[k] = sep_ids[k < n_sep_ids ? k : 0];
  const int threads = scan_threads(S);
  const int chunk = threads * kPer;
  dim3 grid((S + chunk - 1) / chunk, B);
  if (sep::launch_pdl(k_build_index<true>, grid, dim3(threads), 0,
                      static_cast<cudaStream_t>(stream), static_cast<const uint8_t*>(nullptr), ids,
                      set, is_sep, S, prefix, idx, count) != cudaSuccess)
    return SEP_ECUDA;
  return sep::launch_status();
}

extern "C" int sep_count_pairs(const int32_t* prefix, int B, int S, int a, int n,
                               int64_t* kept_pairs, void* stream) {
  if (B < 1 || S < 1 || a < 0 || n < 1) return SEP_EINVAL;
  if (!prefix || !kept_pairs) return SEP_ENULL;
  k_count_pairs<<<B, 1024, 0, static_cast<cudaStream_t>(stream)>>>(prefix, S, a, n, kept_pairs);
  return sep::launch_status();
}
