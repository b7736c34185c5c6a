// The four-block SepCache: bookkeeping, token append and flush compaction.
//
// Blocks (xugj520 SepLLM article, section 3.3 table; KV-manager steps of the
// "HKUDS047: SepLLM ..." study, section "KV Cache Manager"):
//   I  initial cache: the first a tokens, never evicted;
//   S  separator cache: at most s separator tokens, oldest evicted first;
//   P  past window: tokens that slid out of the local window; when it holds
//      more than `past` tokens it is flushed -- its separators join S (which
//      then keeps its newest s entries) and it empties;
//      (variants, the KV manager's switches: without accumulation a flush
//      keeps only P's separators; with an unbounded separator cache an
//      eviction is an error; with the total-length trigger P is flushed when
//      the whole cache holds more than a + s + past + w tokens)
//   L  local window: the newest w tokens.
// Rows of each (layer, b, kv head) are stored I | S | P | L in increasing
// position order.  P and L are one contiguous run of recent positions, so a
// token sliding from L to P moves no data; only a flush moves rows.  A flush
// compacts the surviving rows in place: the survivors are found with an
// order-preserving warp-ballot stream compaction of the I | S | P | L rows,
// so destination row r takes source row src[r] >= r, with src increasing.
// Copying the rows in ascending chunks, every source of a chunk read before
// any destination of that chunk is written, therefore never overwrites a
// row that is still to be read.
//
// Bookkeeping is shared by all layers: sepcache_append at layer 0 runs the
// state machine for the new token and records this step's plan (the row the
// token is written to, the source and destination buffers and, on a flush,
// the source row of every destination row); every layer's append/compact
// (or the fused decode step) then applies that plan to its K/V.
#include <string.h>

#include "common.cuh"

namespace {

// plan[b] = {flush, slot, new_len, nI, -, -, -, -, source row of each
// destination row (flush steps)...}
constexpr int kPlanHdr = 8;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// One warp per sequence.
__global__ void k_cache_advance(int32_t* __restrict__ pos, uint8_t* __restrict__ flag,
                                int32_t* __restrict__ counts, int32_t* __restrict__ plan,
                                int64_t* __restrict__ step, int32_t* __restrict__ status,
                                const uint8_t* __restrict__ is_sep_new, int B, int cap, int a,
                                int s, int past, int w, int mode) {
  const int b = blockIdx.x;
  const int lane = threadIdx.x;
  if (b >= B) return;
  int32_t* cnt = counts + 4 * b;
  int32_t* pl = plan + static_cast<int64_t>(b) * (cap + kPlanHdr);
  int32_t* ps = pos + static_cast<int64_t>(b) * cap;
  uint8_t* fl = flag + static_cast<int64_t>(b) * cap;
  int nI = cnt[0], nS = cnt[1], nP = cnt[2], nL = cnt[3];
  const int64_t t = step[b];
  const uint8_t f = is_sep_new[b] ? 1 : 0;
  int len = nI + nS + nP + nL;
  const bool total_trigger = (mode & SEP_CACHE_TOTAL_TRIGGER) != 0;
  const bool bad = nI < 0 || nS < 0 || nP < 0 || nL < 0 || nI > a || nS > s ||
                   nP > (total_trigger ? past + s : past) || nL > w || len > cap - 1 ||
                   (nI < a && len != nI);
  __syncwarp();
  if (bad) {
    if (lane == 0) {
      atomicOr(status, SEP_CACHE_ESTATE);
      pl[0] = 0;
      pl[1] = -1;
      pl[2] = len > cap ? cap : (len < 0 ? 0 : len);
      pl[3] = 0;
    }
    return;
  }
  // 1. place the token: initial block while it has room, else local window
  const int slot = len;
  if (nI < a) {
    ++nI;
  } else {
    ++nL;
    if (nL > w) {  // the oldest local token now belongs to the past window
      --nL;
      ++nP;
    }
  }
  if (lane == 0) {
    ps[slot] = static_cast<int32_t>(t);
    fl[slot] = f;
  }
  ++len;
  __syncwarp();
  // 2. flush the past window when it overflows (or, with the total-length
  //    trigger, when the whole cache does)
  const bool flush = total_trigger ? len > a + s + past + w : nP > past;
  const bool accumulate = (mode & SEP_CACHE_NO_ACCUMULATION) == 0;
  int new_len = len;
  if (flush) {
    const int eS = nI + nS, eP = eS + nP;
    int ncand = accumulate ? nS : 0;
    for (int base = eS; base < eP; base += 32) {
      const int r = base + lane;
      ncand += __popc(__ballot_sync(0xffffffffu, r < eP && fl[r] != 0));
    }
    const int drop = ncand > s ? ncand - s : 0;
    if (drop > 0 && (mode & SEP_CACHE_UNBOUNDED_SEPS) && lane == 0) atomicOr(status, SEP_CACHE_ESEPS);
    for (int r = lane; r < nI; r += 32) pl[kPlanHdr + r] = r;  // initial rows keep their place
    int rank = 0, dst = nI;
    for (int base = nI; base < len; base += 32) {
      const int r = base + lane;
      const bool valid = r < len;
      const int32_t my_pos = valid ? ps[r] : -1;
      const uint8_t my_flag = valid ? fl[r] : 0;
      const bool is_cand = valid && r < eP && (r < eS ? accumulate : my_flag != 0);
      const bool is_local = valid && r >= eP;
      const uint32_t candb = __ballot_sync(0xffffffffu, is_cand);
      const int my_rank = rank + __popc(candb & lanemask_lt());
      const bool keep = is_local || (is_cand && my_rank >= drop);
      const uint32_t kb = __ballot_sync(0xffffffffu, keep);
      const int d = dst + __popc(kb & lanemask_lt());
      __syncwarp();  // every read of this chunk happens before any write
      if (keep) {
        ps[d] = my_pos;
        fl[d] = my_flag;
        pl[kPlanHdr + d] = r;
      }
      __syncwarp();
      rank += __popc(candb);
      dst += __popc(kb);
    }
    new_len = dst;
    for (int r = new_len + lane; r < len; r += 32) {
      ps[r] = -1;
      fl[r] = 0;
    }
    nS = ncand < s ? ncand : s;
    nP = 0;
    if (new_len != nI + nS + nL && lane == 0) atomicOr(status, SEP_CACHE_ESTATE);
  }
  if (lane == 0) {
    pl[0] = flush ? 1 : 0;
    pl[1] = slot;
    pl[2] = new_len;
    pl[3] = nI;
    cnt[0] = nI;
    cnt[1] = nS;
    cnt[2] = nP;
    cnt[3] = nL;
    step[b] = t + 1;
  }
}

// Byte offset of row 0 of (layer, b, kv head).
__device__ __forceinline__ int64_t row0(int layer, int b, int g, int B, int Hkv, int cap,
                                        int row_bytes) {
  return (((static_cast<int64_t>(layer) * B + b) * Hkv + g) * cap) * row_bytes;
}

// Write the new token's K and V rows of one layer at this step's slot.
__global__ void k_cache_write(uint8_t* __restrict__ kc, uint8_t* __restrict__ vc,
                              const uint8_t* __restrict__ k_new, const uint8_t* __restrict__ v_new,
                              const int32_t* __restrict__ plan, int layer, int B, int Hkv, int cap,
                              int row_bytes) {
  const int b = blockIdx.x;
  const int32_t* pl = plan + static_cast<int64_t>(b) * (cap + kPlanHdr);
  const int slot = pl[1];
  if (slot < 0 || slot >= cap) return;
  const int ch = row_bytes / 16;
  const int per = Hkv * ch;
  for (int e = threadIdx.x; e < 2 * per; e += blockDim.x) {
    const int which = e / per, g = (e % per) / ch, c = e % ch;
    const int64_t dst = row0(layer, b, g, B, Hkv, cap, row_bytes) + static_cast<int64_t>(slot) * row_bytes;
    const int64_t src = (static_cast<int64_t>(b) * Hkv + g) * row_bytes;
    const uint4 val = reinterpret_cast<const uint4*>((which ? v_new : k_new) + src)[c];
    reinterpret_cast<uint4*>((which ? vc : kc) + dst)[c] = val;
  }
}

// Apply this step's flush to one layer, in place: destination row r takes
// source row plan.src[r] >= r (increasing in r).  One CTA per (K or V, kv
// head, b) walks the destination rows in ascending chunks of kChunkRows; it
// reads every source row of a chunk into registers, synchronises, then
// writes the chunk.  A chunk's destinations lie below the sources of every
// later chunk, so nothing is overwritten before it is read.  Rows that do
// not move (the initial block, and any row with src[r] == r) are skipped.
constexpr int kCompactThreads = 256;
constexpr int kCompactUnits = 4;  // 16-byte units per thread and chunk
__global__ void __launch_bounds__(kCompactThreads) k_cache_compact(uint8_t* __restrict__ kc,
                                                                   uint8_t* __restrict__ vc,
                                                                   const int32_t* __restrict__ plan,
                                                                   int layer, int B, int Hkv,
                                                                   int cap, int row_bytes) {
  const int which = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int32_t* pl = plan + static_cast<int64_t>(b) * (cap + kPlanHdr);
  if (pl[0] == 0) return;
  const int new_len = pl[2] < cap ? pl[2] : cap;
  const int first = pl[3] > 0 ? pl[3] : 0;  // the initial rows keep their place
  const int ch = row_bytes / 16;
  const int chunk_rows = kCompactThreads * kCompactUnits / ch;
  uint8_t* base = (which ? vc : kc) + row0(layer, b, g, B, Hkv, cap, row_bytes);
  for (int r0 = first; r0 < new_len; r0 += chunk_rows) {
    uint4 val[kCompactUnits];
    int dst[kCompactUnits];
#pragma unroll
    for (int u = 0; u < kCompactUnits; ++u) {
      const int e = u * kCompactThreads + threadIdx.x;
      const int r = r0 + e / ch, c = e % ch;
      dst[u] = -1;
      if (r < new_len) {
        const int src = pl[kPlanHdr + r];
        if (src >= 0 && src < cap && src != r) {
          val[u] = reinterpret_cast<const uint4*>(base + static_cast<int64_t>(src) * row_bytes)[c];
          dst[u] = r * ch + c;
        }
      }
    }
    __syncthreads();  // every source of the chunk has been read
#pragma unroll
    for (int u = 0; u < kCompactUnits; ++u)
      if (dst[u] >= 0) reinterpret_cast<uint4*>(base)[dst[u]] = val[u];
    __syncthreads();
  }
}

// Prompt ingestion into an empty cache: the state after T sequential
// appends, in closed form.  With nI = min(a, T) initial tokens and nL =
// min(w, T - nI) local ones, E = T - nI - nL tokens left the local window in
// position order and entered the past window, which flushed after every
// past + 1 of them: F = E / (past + 1) flushes took positions [nI, hi), hi =
// nI + F (past + 1), and their separators fed the separator cache, which
// keeps the newest s (the last s separators of [nI, hi) -- a slice of the
// prompt's separator index list); the past window holds [hi, T - nL).  One
// CTA per sequence writes the rows' positions and flags, the block sizes and
// step = T.  A cache that is not empty is left unchanged (status bit).
// Variants: without accumulation the separator cache holds the newest s
// separators of the last flushed block [hi - past - 1, hi) -- again the end
// of the index list up to hi; with the total-length trigger a flush happens
// when the past window exceeds past + s - |S|, so the block ends depend on
// the separator counts and one thread walks them (one step per flush).
__global__ void k_cache_ingest_meta(int32_t* __restrict__ pos, uint8_t* __restrict__ flag,
                                    int32_t* __restrict__ counts, int32_t* __restrict__ plan,
                                    int64_t* __restrict__ step, int32_t* __restrict__ status,
                                    const uint8_t* __restrict__ is_sep,
                                    const int32_t* __restrict__ prefix,
                                    const int32_t* __restrict__ idx, int T, int cap, int a, int s,
                                    int past, int w, int mode) {
  __shared__ int empty, sh_hi, sh_ns, sh_ovf;
  const int b = blockIdx.x;
  int32_t* cnt = counts + 4 * b;
  if (threadIdx.x == 0)
    empty = step[b] == 0 && cnt[0] == 0 && cnt[1] == 0 && cnt[2] == 0 && cnt[3] == 0;
  __syncthreads();
  if (!empty) {
    if (threadIdx.x == 0) atomicOr(status, SEP_CACHE_ESTATE);
    return;
  }
  const uint8_t* f = is_sep + static_cast<int64_t>(b) * T;
  const int32_t* pre = prefix + static_cast<int64_t>(b) * (T + 1);
  const int32_t* ix = idx + static_cast<int64_t>(b) * T;
  const int nI = a < T ? a : T;
  const int rest = T - nI;
  const int nL = w < rest ? w : rest;
  const int E = rest - nL;
  const bool accumulate = (mode & SEP_CACHE_NO_ACCUMULATION) == 0;
  if (threadIdx.x == 0) {
    int hi = nI, ns = 0, ovf = 0;
    if (mode & SEP_CACHE_TOTAL_TRIGGER) {
      // the k-th flush takes the past window once it holds past + s - |S| + 1
      for (;;) {
        const int blen = past + s - ns + 1;
        if (hi + blen > nI + E) break;
        const int cnt = pre[hi + blen] - pre[hi];
        const int cand = (accumulate ? ns : 0) + cnt;
        ovf |= cand > s;
        ns = cand < s ? cand : s;
        hi += blen;
      }
    } else {
      const int F = E / (past + 1);
      hi = nI + F * (past + 1);
      if (F > 0) {
        const int cand = accumulate ? pre[hi] - pre[nI] : pre[hi] - pre[hi - past - 1];
        ns = cand < s ? cand : s;
        if (accumulate) {
          ovf = cand > s;
        } else {
          for (int k = 0; k < F && !ovf; ++k)
            ovf = pre[nI + (k + 1) * (past + 1)] - pre[nI + k * (past + 1)] > s;
        }
      }
    }
    sh_hi = hi;
    sh_ns = ns;
    sh_ovf = ovf;
  }
  __syncthreads();
  const int hi = sh_hi;
  const int nS = sh_ns;
  const int nP = E - (hi - nI);
  if (sh_ovf && (mode & SEP_CACHE_UNBOUNDED_SEPS) && threadIdx.x == 0) atomicOr(status, SEP_CACHE_ESEPS);
  const int len = nI + nS + nP + nL;
  const int s0 = pre[hi] - nS;  // index-list entry of the oldest kept separator
  const int l0 = T - nL;
  int32_t* ps = pos + static_cast<int64_t>(b) * cap;
  uint8_t* fl = flag + static_cast<int64_t>(b) * cap;
  for (int r = threadIdx.x; r < cap; r += blockDim.x) {
    int p = -1;
    if (r < nI) p = r;
    else if (r < nI + nS) p = ix[s0 + (r - nI)];
    else if (r < nI + nS + nP) p = hi + (r - nI - nS);
    else if (r < len) p = l0 + (r - nI - nS - nP);
    uint8_t fv = 0;
    if (p >= T || (p < 0 && r < len)) {
      atomicOr(status, SEP_CACHE_ESTATE);
      p = -1;
    } else if (p >= 0) {
      fv = f[p] ? 1 : 0;
    }
    ps[r] = p;
    fl[r] = fv;
  }
  if (threadIdx.x == 0) {
    cnt[0] = nI;
    cnt[1] = nS;
    cnt[2] = nP;
    cnt[3] = nL;
    step[b] = T;
    int32_t* pl = plan + static_cast<int64_t>(b) * (cap + kPlanHdr);
    pl[0] = 0;
    pl[1] = -1;
    pl[2] = len;
    pl[3] = nI;
    pl[4] = pl[5] = 0;
    pl[6] = pl[7] = 0;
  }
}

// One layer's K/V rows of an ingested prompt: row r takes the
// prompt's row at position pos[r] (k, v: [B][Hkv][T][D]).  Grid: (chunks,
// kv head, b).  Skips a sequence whose ingestion did not happen (step != T).
__global__ void __launch_bounds__(256) k_cache_ingest_rows(
    uint8_t* __restrict__ kc, uint8_t* __restrict__ vc, const uint8_t* __restrict__ k,
    const uint8_t* __restrict__ v, const int32_t* __restrict__ pos,
    const int32_t* __restrict__ counts, const int64_t* __restrict__ step, int T, int layer, int B,
    int Hkv, int cap, int row_bytes) {
  const int g = blockIdx.y, b = blockIdx.z;
  if (step[b] != T) return;
  const int32_t* cnt = counts + 4 * b;
  const int len = cnt[0] + cnt[1] + cnt[2] + cnt[3];
  if (len < 0 || len > cap) return;
  const int ch = row_bytes / 16;  // 16-byte chunks per row: a power of two (8, 16 or 32)
  const int lg = __ffs(ch) - 1;
  const int64_t dbase = row0(layer, b, g, B, Hkv, cap, row_bytes);
  const int64_t sbase = (static_cast<int64_t>(b) * Hkv + g) * T * row_bytes;
  const int32_t* ps = pos + static_cast<int64_t>(b) * cap;
  const int half = len << lg;  // chunks of K; V follows
  // one chunk per thread, the K rows first, then the V rows (shifts and a
  // compare, no division)
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < 2 * half; e += gridDim.x * blockDim.x) {
    const bool which = e >= half;
    const int e1 = which ? e - half : e;
    const int r = e1 >> lg, c = e1 & (ch - 1);
    const int p = ps[r];
    if (p < 0 || p >= T) continue;
    const uint4 val = reinterpret_cast<const uint4*>((which ? v : k) + sbase + static_cast<int64_t>(p) * row_bytes)[c];
    reinterpret_cast<uint4*>((which ? vc : kc) + dbase + static_cast<int64_t>(r) * row_bytes)[c] = val;
  }
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

struct Sizes {
  size_t k, v, pos, flag, counts, plan, step, status, rope;
  size_t total() const { return k + v + pos + flag + counts + plan + step + status + rope; }
};

// rows of the rotary table: every slot, and at least 65 so that the decode
// kernels can read the turns by 8 and by 64 slots
int rope_rows_of(int64_t cap) { return static_cast<int>(cap > 65 ? cap : 65); }

Sizes sizes(sep_cache_cfg cfg, int layers, int B, int Hkv, int D, int dtype) {
  const int64_t cap = static_cast<int64_t>(cfg.a) + cfg.s + cfg.past + cfg.w + 1;
  Sizes z;
  z.k = round256(static_cast<size_t>(layers) * B * Hkv * cap * D * sep::elem_bytes(dtype));
  z.v = z.k;
  z.pos = round256(static_cast<size_t>(B) * cap * 4);
  z.flag = round256(static_cast<size_t>(B) * cap);
  z.counts = round256(static_cast<size_t>(B) * 16);
  z.plan = round256(static_cast<size_t>(B) * (cap + kPlanHdr) * 4);
  z.step = round256(static_cast<size_t>(B) * 8);
  z.status = 256;
  z.rope = round256(static_cast<size_t>(rope_rows_of(cap)) * D * 4);
  return z;
}

bool cfg_ok(sep_cache_cfg cfg, int layers, int B, int Hkv, int D, int dtype) {
  if (cfg.a < 0 || cfg.s < 0 || cfg.past < 0 || cfg.w < 1 || (cfg.mode & ~7) != 0) return false;
  if (layers < 1 || B < 1 || Hkv < 1 || B > 65535) return false;
  if (dtype != SEP_F32 && dtype != SEP_BF16) return false;
  if (D != 64 && D != 128) return false;
  const int64_t cap = static_cast<int64_t>(cfg.a) + cfg.s + cfg.past + cfg.w + 1;
  return cap < (1 << 20);
}

bool cache_ok(const sepcache* c) {
  return c && c->k && c->v && c->pos && c->flag && c->counts && c->plan && c->step && c->status &&
         c->rope && c->rope_rows == rope_rows_of(c->cap) && c->rope_theta >= 0.f &&
         cfg_ok(c->cfg, c->layers, c->B, c->Hkv, c->D, c->dtype) &&
         c->cap == c->cfg.a + c->cfg.s + c->cfg.past + c->cfg.w + 1;
}

}  // namespace

extern "C" size_t sepcache_bytes(sep_cache_cfg cfg, int layers, int B, int Hkv, int D, int dtype) {
  if (!cfg_ok(cfg, layers, B, Hkv, D, dtype)) return 0;
  return sizes(cfg, layers, B, Hkv, D, dtype).total();
}

extern "C" int sepcache_carve(sepcache* cache, void* buffer, size_t bytes, sep_cache_cfg cfg,
                              int layers, int B, int Hkv, int D, int dtype) {
  if (!cache || !buffer) return SEP_ENULL;
  if (!cfg_ok(cfg, layers, B, Hkv, D, dtype)) {
    if (dtype != SEP_F32 && dtype != SEP_BF16) return SEP_EDTYPE;
    if (D != 64 && D != 128) return SEP_EDTYPE;
    return SEP_EINVAL;
  }
  if ((reinterpret_cast<uintptr_t>(buffer) & 255u) != 0) return SEP_EALIGN;
  const Sizes z = sizes(cfg, layers, B, Hkv, D, dtype);
  if (bytes < z.total()) return SEP_EINVAL;
  uint8_t* p = static_cast<uint8_t*>(buffer);
  memset(cache, 0, sizeof *cache);
  cache->k = p;
  p += z.k;
  cache->v = p;
  p += z.v;
  cache->pos = reinterpret_cast<int32_t*>(p);
  p += z.pos;
  cache->flag = p;
  p += z.flag;
  cache->counts = reinterpret_cast<int32_t*>(p);
  p += z.counts;
  cache->plan = reinterpret_cast<int32_t*>(p);
  p += z.plan;
  cache->step = reinterpret_cast<int64_t*>(p);
  p += z.step;
  cache->status = reinterpret_cast<int32_t*>(p);
  p += z.status;
  cache->rope = reinterpret_cast<float*>(p);
  cache->layers = layers;
  cache->B = B;
  cache->Hkv = Hkv;
  cache->D = D;
  cache->dtype = dtype;
  cache->cap = cfg.a + cfg.s + cfg.past + cfg.w + 1;
  cache->cfg = cfg;
  cache->rope_theta = 0.f;
  cache->rope_rows = rope_rows_of(cache->cap);
  return SEP_OK;
}

namespace {
// cos / sin of slot r at frequency i: phi = r * theta^(-2i/D), evaluated in
// fp64 and rounded to fp32
__global__ void k_rope_table(float* tab, int rows, int D, double theta) {
  const int half = D / 2;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= rows * half) return;
  const int r = e / half, i = e % half;
  const double phi = static_cast<double>(r) * pow(theta, -2.0 * i / D);
  double sn, cs;
  sincos(phi, &sn, &cs);
  tab[2 * e] = static_cast<float>(cs);
  tab[2 * e + 1] = static_cast<float>(sn);
}
}  // namespace

extern "C" int sepcache_set_rope(sepcache* c, float theta, void* stream) {
  if (!c) return SEP_ENULL;
  if (!cache_ok(c)) return SEP_EINVAL;
  if (!(theta >= 0.f) || !isfinite(theta) || (theta > 0.f && theta <= 1.f)) return SEP_EINVAL;
  if (theta == 0.f) {
    c->rope_theta = 0.f;
    return SEP_OK;
  }
  const int n = c->rope_rows * (c->D / 2);
  k_rope_table<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      c->rope, c->rope_rows, c->D, static_cast<double>(theta));
  const int rc = sep::launch_status();
  if (rc == SEP_OK) c->rope_theta = theta;
  return rc;
}

extern "C" int sepcache_init(const sepcache* c, void* stream) {
  if (!cache_ok(c)) return c ? SEP_EINVAL : SEP_ENULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t cap = static_cast<size_t>(c->cap);
  bool ok = cudaMemsetAsync(c->pos, 0xff, c->B * cap * 4, st) == cudaSuccess &&
            cudaMemsetAsync(c->flag, 0, c->B * cap, st) == cudaSuccess &&
            cudaMemsetAsync(c->counts, 0, c->B * 16, st) == cudaSuccess &&
            cudaMemsetAsync(c->plan, 0, c->B * (cap + kPlanHdr) * 4, st) == cudaSuccess &&
            cudaMemsetAsync(c->step, 0, c->B * 8, st) == cudaSuccess &&
            cudaMemsetAsync(c->status, 0, 4, st) == cudaSuccess;
  return ok ? SEP_OK : SEP_ECUDA;
}

namespace sep {
int cache_advance(const sepcache* c, const uint8_t* is_sep_new, cudaStream_t st) {
  // A plain launch, and it must stay one (no programmatic stream
  // serialization): it starts only after every kernel of the previous step
  // has completed, which is what lets the fused decode of layers >= 1 read
  // the cache metadata and its layer's rows before its grid-dependency wait.
  k_cache_advance<<<c->B, 32, 0, st>>>(c->pos, c->flag, c->counts, c->plan, c->step, c->status,
                                        is_sep_new, c->B, c->cap, c->cfg.a, c->cfg.s, c->cfg.past,
                                        c->cfg.w, c->cfg.mode);
  return launch_status();
}
bool cache_valid(const sepcache* c) { return cache_ok(c); }
}  // namespace sep

extern "C" int sepcache_append(const sepcache* c, int layer, const void* k_new, const void* v_new,
                               const uint8_t* is_sep_new, void* stream) {
  if (!cache_ok(c)) return c ? SEP_EINVAL : SEP_ENULL;
  if (layer < 0 || layer >= c->layers) return SEP_EINVAL;
  if (!k_new || !v_new || (layer == 0 && !is_sep_new)) return SEP_ENULL;
  if (!sep::aligned16(k_new) || !sep::aligned16(v_new)) return SEP_EALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (layer == 0) {
    // a plain launch (no programmatic serialization), as in cache_advance
    k_cache_advance<<<c->B, 32, 0, st>>>(c->pos, c->flag, c->counts, c->plan, c->step, c->status,
                                          is_sep_new, c->B, c->cap, c->cfg.a, c->cfg.s, c->cfg.past,
                                          c->cfg.w, c->cfg.mode);
    if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  }
  const int row_bytes = c->D * sep::elem_bytes(c->dtype);
  const int threads = 2 * c->Hkv * row_bytes / 16 < 512 ? 2 * c->Hkv * row_bytes / 16 : 512;
  k_cache_write<<<c->B, (threads + 31) / 32 * 32, 0, st>>>(
      static_cast<uint8_t*>(c->k), static_cast<uint8_t*>(c->v),
      static_cast<const uint8_t*>(k_new), static_cast<const uint8_t*>(v_new), c->plan, layer, c->B,
      c->Hkv, c->cap, row_bytes);
  return sep::launch_status();
}

extern "C" int sepcache_compact(const sepcache* c, int layer, void* stream) {
  if (!cache_ok(c)) return c ? SEP_EINVAL : SEP_ENULL;
  if (layer < 0 || layer >= c->layers) return SEP_EINVAL;
  const int row_bytes = c->D * sep::elem_bytes(c->dtype);
  dim3 grid(2, c->Hkv, c->B);
  k_cache_compact<<<grid, kCompactThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint8_t*>(c->k), static_cast<uint8_t*>(c->v), c->plan, layer, c->B, c->Hkv,
      c->cap, row_bytes);
  return sep::launch_status();
}

extern "C" int sepcache_ingest(const sepcache* c, int layer, const void* k, const void* v,
                               const uint8_t* is_sep, const int32_t* prefix, const int32_t* idx,
                               int T, void* stream) {
  if (!cache_ok(c)) return c ? SEP_EINVAL : SEP_ENULL;
  if (layer < 0 || layer >= c->layers || T < 1) return SEP_EINVAL;
  if (!k || !v || (layer == 0 && (!is_sep || !prefix || !idx))) return SEP_ENULL;
  if (!sep::aligned16(k) || !sep::aligned16(v)) return SEP_EALIGN;
  if (static_cast<int64_t>(c->B) * c->Hkv * T >= (1ll << 31)) return SEP_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (layer == 0) {
    k_cache_ingest_meta<<<c->B, 256, 0, st>>>(c->pos, c->flag, c->counts, c->plan, c->step,
                                               c->status, is_sep, prefix, idx, T, c->cap,
                                               c->cfg.a, c->cfg.s, c->cfg.past, c->cfg.w, c->cfg.mode);
    if (cudaGetLastError() != cudaSuccess) return SEP_ECUDA;
  }
  const int row_bytes = c->D * sep::elem_bytes(c->dtype);
  // one 16-byte chunk per thread for a full cache: the copy is a chain of
  // dependent loads (row position, then data), so width hides its latency
  const int chunks = 2 * c->cap * (row_bytes / 16);
  dim3 grid((chunks + 255) / 256, c->Hkv, c->B);
  k_cache_ingest_rows<<<grid, 256, 0, st>>>(
      static_cast<uint8_t*>(c->k), static_cast<uint8_t*>(c->v), static_cast<const uint8_t*>(k),
      static_cast<const uint8_t*>(v), c->pos, c->counts, c->step, T, layer, c->B, c->Hkv, c->cap,
      row_bytes);
  return sep::launch_status();
}

extern "C" int sepcache_status(const sepcache* c, int32_t* host_status, void* stream) {
  if (!c || !c->status) return SEP_ENULL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, c->status, 4, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return SEP_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SEP_ECUDA;
  if (host_status) *host_status = v;
  return v ? SEP_EDEVICE : SEP_OK;
}
