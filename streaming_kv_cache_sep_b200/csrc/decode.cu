// Decode attention of the newest token over the SepCache (split-K, GQA-aware).
//
// The cache keeps only the initial, separator, past-window and local-window
// rows, so a decode step reads len[b] <= a + s + past + w K/V rows per
// (sequence, kv head) (jieyibu.net explainer, section 1.3: fewer KV pairs to
// load).  The kernel is bound by HBM bandwidth:
//   * grid (split, kv head, sequence); a CTA takes 64 consecutive rows of one
//     (b, kv head) and pulls them into shared memory with two bulk copies
//     (K and V, one mbarrier), so each byte is read from HBM once per step;
//   * the G = Hq/Hkv query heads of the group share every K/V row;
//   * each CTA writes an unnormalised partial (max, sum, G x D output); the
//     last CTA of a (b, kv head) to finish (an atomic ticket, no waiting)
//     merges the partials and writes out and lse.
#include "common.cuh"

namespace {

constexpr int ROWS = 64;  // rows per split
constexpr int kThreads = 128;

template <typename T>
__device__ __forceinline__ float to_f(T x);
template <>
__device__ __forceinline__ float to_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f(float x);
template <>
__device__ __forceinline__ float from_f<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// DPL consecutive elements of a row starting at element d0, as floats.
template <typename T, int DPL>
__device__ __forceinline__ void load_row_slice(const T* row, int d0, float (&x)[DPL]) {
#pragma unroll
  for (int e = 0; e < DPL; ++e) x[e] = to_f(row[d0 + e]);
}

struct DecodeParams {
  const void* q;
  const void* kc;
  const void* vc;
  const int32_t* counts;
  void* out;
  float* lse;
  float* part_ml;  // [B][Hq][nsplit][2]
  float* part_o;   // [B][Hq][nsplit][D]
  int32_t* ticket; // [B][Hkv]
  int32_t* err;
  int layer, B, Hq, Hkv, cap, nsplit;
  float scale_log2;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads) k_decode(const DecodeParams p) {
  constexpr int DPL = D / 32;
  // dynamic: K rows | V rows; the cross-warp reduction reuses the K rows
  extern __shared__ __align__(128) uint8_t dsm[];
  T* sk = reinterpret_cast<T*>(dsm);
  T* sv = sk + ROWS * D;
  float(*red)[G][D] = reinterpret_cast<float(*)[G][D]>(dsm);
  static_assert(sizeof(T) * ROWS * D >= sizeof(float) * 4 * G * D, "reduction must fit in K rows");
  __shared__ float sq[G][D];
  __shared__ float ss[G][ROWS];
  __shared__ float sm[G], sl[G];
  __shared__ __align__(8) uint64_t bar;
  __shared__ int is_last;
  __shared__ int abort_flag;

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* cnt = p.counts + 4 * b;
  const int len = cnt[0] + cnt[1] + cnt[2] + cnt[3];
  const int r0 = split * ROWS;
  if (len <= 0 || len > p.cap || r0 >= len) return;
  const int nrows = len - r0 < ROWS ? len - r0 : ROWS;
  const int nsplit_b = (len + ROWS - 1) / ROWS;

  const int64_t kv_base =
      ((static_cast<int64_t>(p.layer) * p.B + b) * p.Hkv + g) * p.cap * D + static_cast<int64_t>(r0) * D;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sep::mbar_init(&bar, 1);
    sep::mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t bytes = static_cast<uint32_t>(nrows * D * sizeof(T));
    sep::mbar_arrive_expect_tx(&bar, 2 * bytes);
    sep::bulk_load(sk, static_cast<const T*>(p.kc) + kv_base, bytes, &bar);
    sep::bulk_load(sv, static_cast<const T*>(p.vc) + kv_base, bytes, &bar);
  }
  // query rows of the group's heads, pre-scaled into the log2 domain
  const T* qg = static_cast<const T*>(p.q) + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
  for (int e = threadIdx.x; e < G * D; e += kThreads) sq[e / D][e % D] = to_f(qg[e]) * p.scale_log2;
  __syncthreads();
  const bool landed = sep::mbar_wait(&bar, 0, &abort_flag, p.err);
  if (!landed) {  // the copies must land before this CTA's shared memory is reused
    int keep_waiting = 0;
    sep::mbar_wait(&bar, 0, &keep_waiting, nullptr);
  }

  // scores: warp w takes rows w, w+4, ...; lane owns DPL consecutive dims
  const int d0 = lane * DPL;
  float qv[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) qv[h][e] = sq[h][d0 + e];
  if (landed) {
    for (int r = warp; r < nrows; r += 4) {
      float x[DPL];
      load_row_slice<T, DPL>(sk + r * D, d0, x);
      float acc[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < DPL; ++e) a = fmaf(qv[h][e], x[e], a);
        acc[h] = a;
      }
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int o = 16; o; o >>= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], o);
      if (lane < G) {
        float v = acc[0];
#pragma unroll
        for (int h = 1; h < G; ++h)
          if (lane == h) v = acc[h];
        ss[lane][r] = v;
      }
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
  // P V: warp-private accumulators, then a cross-warp sum
  float o[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) o[h][e] = 0.f;
  if (landed) {
    for (int r = warp; r < nrows; r += 4) {
      float x[DPL];
      load_row_slice<T, DPL>(sv + r * D, d0, x);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float pr = ss[h][r];
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[h][e] = fmaf(pr, x[e], o[h][e]);
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int e = 0; e < DPL; ++e) red[warp][h][d0 + e] = o[h][e];  // K rows are no longer read
  __syncthreads();

  T* out = static_cast<T*>(p.out);
  const int hq0 = g * G;
  if (nsplit_b == 1) {
    for (int e = threadIdx.x; e < G * D; e += kThreads) {
      const int h = e / D, d = e % D;
      const float s = red[0][h][d] + red[1][h][d] + red[2][h][d] + red[3][h][d];
      out[(static_cast<int64_t>(b) * p.Hq + hq0 + h) * D + d] = from_f<T>(s / sl[h]);
    }
    if (p.lse && threadIdx.x < G)
      p.lse[static_cast<int64_t>(b) * p.Hq + hq0 + threadIdx.x] =
          (sm[threadIdx.x] + log2f(sl[threadIdx.x])) * 0.69314718055994530942f;
    return;
  }
  // write this split's partial
  for (int e = threadIdx.x; e < G * D; e += kThreads) {
    const int h = e / D, d = e % D;
    const float s = red[0][h][d] + red[1][h][d] + red[2][h][d] + red[3][h][d];
    p.part_o[((static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit + split) * D + d] = s;
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
  if (!is_last) return;
  __threadfence();
  // merge the partials of every split of this (b, kv head)
  for (int h = warp; h < G; h += 4) {
    const float* ml = p.part_ml + (static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit * 2;
    float M = -INFINITY;
    for (int s = 0; s < nsplit_b; ++s) M = fmaxf(M, __ldcg(ml + 2 * s));
    float Lsum = 0.f;
    for (int s = 0; s < nsplit_b; ++s) Lsum += __ldcg(ml + 2 * s + 1) * exp2f(__ldcg(ml + 2 * s) - M);
    const float* po = p.part_o + (static_cast<int64_t>(b) * p.Hq + hq0 + h) * p.nsplit * D;
    for (int d = lane; d < D; d += 32) {
      float acc = 0.f;
      for (int s = 0; s < nsplit_b; ++s) acc += __ldcg(po + s * D + d) * exp2f(__ldcg(ml + 2 * s) - M);
      out[(static_cast<int64_t>(b) * p.Hq + hq0 + h) * D + d] = from_f<T>(acc / Lsum);
    }
    if (p.lse && lane == 0)
      p.lse[static_cast<int64_t>(b) * p.Hq + hq0 + h] = (M + log2f(Lsum)) * 0.69314718055994530942f;
  }
}

template <typename T, int D, int G>
int launch_one(const DecodeParams& p, cudaStream_t st) {
  constexpr int smem = 2 * ROWS * D * static_cast<int>(sizeof(T));
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (smem > 48 * 1024 && dev >= 0 && dev < 64 && !attr_set[dev]) {
    if (cudaFuncSetAttribute(k_decode<T, D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return SEP_ECUDA;
    attr_set[dev] = true;
  }
  dim3 grid(p.nsplit, p.Hkv, p.B);
  k_decode<T, D, G><<<grid, kThreads, smem, st>>>(p);
  return sep::launch_status();
}

template <typename T, int D>
int launch_g(const DecodeParams& p, int G, cudaStream_t st) {
  switch (G) {
    case 1: return launch_one<T, D, 1>(p, st);
    case 2: return launch_one<T, D, 2>(p, st);
    case 4: return launch_one<T, D, 4>(p, st);
    case 8: return launch_one<T, D, 8>(p, st);
    default: return SEP_EINVAL;
  }
}

bool cache_ok(const sepcache* c) {
  return c && c->k && c->v && c->counts && c->cap == c->cfg.a + c->cfg.s + c->cfg.past + c->cfg.w + 1 &&
         c->layers >= 1 && c->B >= 1 && c->Hkv >= 1 && (c->D == 64 || c->D == 128) &&
         (c->dtype == SEP_F32 || c->dtype == SEP_BF16);
}

struct WsLayout {
  size_t ml, o, ticket;
};
WsLayout ws_layout(const sepcache* c, int Hq) {
  const size_t nsplit = (c->cap + ROWS - 1) / ROWS;
  WsLayout w;
  w.ml = (static_cast<size_t>(c->B) * Hq * nsplit * 2 * 4 + 255) / 256 * 256;
  w.o = (static_cast<size_t>(c->B) * Hq * nsplit * c->D * 4 + 255) / 256 * 256;
  w.ticket = (static_cast<size_t>(c->B) * c->Hkv * 4 + 255) / 256 * 256;
  return w;
}

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
  DecodeParams p;
  p.q = q;
  p.kc = c->k;
  p.vc = c->v;
  p.counts = c->counts;
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
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c->dtype == SEP_BF16)
    return c->D == 64 ? launch_g<__nv_bfloat16, 64>(p, G, st) : launch_g<__nv_bfloat16, 128>(p, G, st);
  return c->D == 64 ? launch_g<float, 64>(p, G, st) : launch_g<float, 128>(p, G, st);
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
namespace {

constexpr int kNoAllocMaxPartials = 8192;  // B * Hq * splits, splits = ceil(cap / 64)
constexpr int kNoAllocMaxTickets = 4096;   // B * Hkv
constexpr size_t kNoAllocMlBytes = static_cast<size_t>(kNoAllocMaxPartials) * 2 * 4;
constexpr size_t kNoAllocOBytes = static_cast<size_t>(kNoAllocMaxPartials) * 128 * 4;
constexpr size_t kNoAllocTicketBytes = static_cast<size_t>(kNoAllocMaxTickets) * 4;
constexpr size_t kNoAllocBytes = kNoAllocMlBytes + kNoAllocOBytes + kNoAllocTicketBytes;

__device__ __align__(256) uint8_t g_decode_scratch[kNoAllocBytes];

constexpr int kNoAllocMaxDevices = 64;
uint8_t* g_decode_scratch_addr[kNoAllocMaxDevices];  // device address, per device

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
  if (static_cast<int64_t>(c->B) * Hq * nsplit > kNoAllocMaxPartials ||
      static_cast<int64_t>(c->B) * c->Hkv > kNoAllocMaxTickets)
    return SEP_ETOOBIG;
  // set-up, once per device with that device current: the device address of
  // the scratch array (the host-side symbol itself is not a device address)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return SEP_ECUDA;
  if (!g_decode_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return SEP_ECUDA;
    g_decode_scratch_addr[dev] = static_cast<uint8_t*>(p);
  }
  uint8_t* scratch = g_decode_scratch_addr[dev];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* tickets = reinterpret_cast<int32_t*>(scratch + kNoAllocMlBytes + kNoAllocOBytes);
  // the tickets must start at zero (the array keeps the previous call's contents)
  if (cudaMemsetAsync(tickets, 0, static_cast<size_t>(c->B) * c->Hkv * 4, st) != cudaSuccess)
    return SEP_ECUDA;
  DecodeParams p;
  p.q = q;
  p.kc = c->k;
  p.vc = c->v;
  p.counts = c->counts;
  p.out = out;
  p.lse = lse;
  p.part_ml = reinterpret_cast<float*>(scratch);
  p.part_o = reinterpret_cast<float*>(scratch + kNoAllocMlBytes);
  p.ticket = tickets;
  p.err = sep::device_error_word();
  p.layer = layer;
  p.B = c->B;
  p.Hq = Hq;
  p.Hkv = c->Hkv;
  p.cap = c->cap;
  p.nsplit = nsplit;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(c->D));
  p.scale_log2 = sc * 1.44269504088896340736f;
  if (c->dtype == SEP_BF16)
    return c->D == 64 ? launch_g<__nv_bfloat16, 64>(p, G, st) : launch_g<__nv_bfloat16, 128>(p, G, st);
  return c->D == 64 ? launch_g<float, 64>(p, G, st) : launch_g<float, 128>(p, G, st);
}
