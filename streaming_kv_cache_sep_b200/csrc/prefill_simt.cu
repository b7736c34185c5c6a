// Exact-fp32 Sep-Attention prefill on the FMA pipes (fp32 inputs).
//
// One warp owns one query row i of one head.  Its kept keys are enumerated in
// three runs -- initial tokens [0, min(a, lo)), separators in [a, lo) taken
// from the index list, and the window [lo, i] with lo = max(0, i - n + 1) --
// which is exactly {j <= i : j < a or is_sep[j] or i - j < n}, each key once
// ("HKUDS047: SepLLM ..." study, section "SepAttention").  Keys are scored
// 32 at a time (lane = key), with an online softmax; the output row is
// accumulated with lane = head dimension.  TF32 tensor cores cannot meet an
// fp32 tolerance, so this path stays on FFMA.
#include "common.cuh"

namespace {

template <int D>
__global__ void __launch_bounds__(128) k_prefill_f32(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const int32_t* __restrict__ prefix, const int32_t* __restrict__ idx, int B, int Hq, int Hkv,
    int S, int a, int n, float scale_log2, float* __restrict__ out, float* __restrict__ lse) {
  constexpr int DPL = D / 32;  // output dims per lane
  __shared__ float qs[4][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;  // (b*Hq + h)*S + i
  const int64_t nrows = static_cast<int64_t>(B) * Hq * S;
  if (row >= nrows) return;
  const int i = static_cast<int>(row % S);
  const int64_t bh = row / S;
  const int h = static_cast<int>(bh % Hq);
  const int b = static_cast<int>(bh / Hq);
  const int g = h / (Hq / Hkv);

  for (int d = lane; d < D; d += 32) qs[warp][d] = q[row * D + d];
  __syncwarp();

  const int32_t* pre = prefix + static_cast<int64_t>(b) * (S + 1);
  const int32_t* ix = idx + static_cast<int64_t>(b) * S;
  const int lo = i - n + 1 > 0 ? i - n + 1 : 0;
  const int n_init = a < lo ? a : lo;
  const int aa = a < S ? a : S;
  const int sep_begin = pre[aa];
  const int n_sep = lo > aa ? pre[lo] - sep_begin : 0;
  const int n_win = i - lo + 1;
  const int nk = n_init + n_sep + n_win;

  const float* kb = k + static_cast<int64_t>(b * Hkv + g) * S * D;
  const float* vb = v + static_cast<int64_t>(b * Hkv + g) * S * D;

  float m = -INFINITY, l = 0.f;
  float acc[DPL];
#pragma unroll
  for (int r = 0; r < DPL; ++r) acc[r] = 0.f;

  for (int c0 = 0; c0 < nk; c0 += 32) {
    const int t = c0 + lane;
    int pos = -1;
    if (t < nk) {
      if (t < n_init)
        pos = t;
      else if (t < n_init + n_sep)
        pos = ix[sep_begin + (t - n_init)];
      else
        pos = lo + (t - n_init - n_sep);
    }
    float s = -INFINITY;
    if (pos >= 0) {
      const float4* kr = reinterpret_cast<const float4*>(kb + static_cast<int64_t>(pos) * D);
      float dot = 0.f;
#pragma unroll 8
      for (int d4 = 0; d4 < D / 4; ++d4) {
        float4 x = kr[d4];
        dot = fmaf(qs[warp][4 * d4 + 0], x.x, dot);
        dot = fmaf(qs[warp][4 * d4 + 1], x.y, dot);
        dot = fmaf(qs[warp][4 * d4 + 2], x.z, dot);
        dot = fmaf(qs[warp][4 * d4 + 3], x.w, dot);
      }
      s = dot * scale_log2;  // log2-domain score
    }
    float cm = s;
    for (int o = 16; o; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
    const float m_new = fmaxf(m, cm);
    const float alpha = exp2f(m - m_new);  // 0 on the first chunk
    const float p = pos >= 0 ? exp2f(s - m_new) : 0.f;
    float ps = p;
    for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * alpha + ps;
#pragma unroll
    for (int r = 0; r < DPL; ++r) acc[r] *= alpha;
    const int cnt = nk - c0 < 32 ? nk - c0 : 32;
    for (int u = 0; u < cnt; ++u) {
      const float pu = __shfl_sync(0xffffffffu, p, u);
      const int posu = __shfl_sync(0xffffffffu, pos, u);
      const float* vr = vb + static_cast<int64_t>(posu) * D;
#pragma unroll
      for (int r = 0; r < DPL; ++r) acc[r] = fmaf(pu, vr[lane + 32 * r], acc[r]);
    }
    m = m_new;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int r = 0; r < DPL; ++r) out[row * D + lane + 32 * r] = acc[r] * inv;
  if (lse && lane == 0) lse[row] = (m + log2f(l)) * 0.69314718055994530942f;
}

}  // namespace

namespace sep {
int prefill_f32(const float* q, const float* k, const float* v, const int32_t* prefix,
                const int32_t* idx, int B, int Hq, int Hkv, int S, int D, int a, int n,
                float scale, float* out, float* lse, cudaStream_t st) {
  const float scale_log2 = scale * 1.44269504088896340736f;
  const int64_t rows = static_cast<int64_t>(B) * Hq * S;
  const int64_t blocks = (rows + 3) / 4;
  if (blocks > 0x7fffffff) return SEP_EINVAL;
  switch (D) {
    case 32:
      k_prefill_f32<32><<<static_cast<unsigned>(blocks), 128, 0, st>>>(
          q, k, v, prefix, idx, B, Hq, Hkv, S, a, n, scale_log2, out, lse);
      break;
    case 64:
      k_prefill_f32<64><<<static_cast<unsigned>(blocks), 128, 0, st>>>(
          q, k, v, prefix, idx, B, Hq, Hkv, S, a, n, scale_log2, out, lse);
      break;
    case 128:
      k_prefill_f32<128><<<static_cast<unsigned>(blocks), 128, 0, st>>>(
          q, k, v, prefix, idx, B, Hq, Hkv, S, a, n, scale_log2, out, lse);
      break;
    default:
      return SEP_EDTYPE;
  }
  return launch_status();
}
}  // namespace sep
