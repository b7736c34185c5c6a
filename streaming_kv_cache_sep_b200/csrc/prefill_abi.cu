// C-ABI entry of the prefill: argument checks and dtype dispatch.
#include <math.h>

#include "common.cuh"
#include "internal.h"

extern "C" size_t sep_attn_prefill_workspace(int B, int Hq, int Hkv, int S, int D, int dtype) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || D < 1) return 0;
  if (dtype == SEP_BF16) return sep::prefill_tc_workspace(B, Hkv, S, D);
  return 256;
}

extern "C" int sep_attn_prefill(const void* q, const void* k, const void* v, int dtype,
                                const uint8_t* is_sep, const int32_t* prefix, const int32_t* idx,
                                int B, int Hq, int Hkv, int S, int D, int a, int n, float scale,
                                void* out, float* lse, void* workspace, size_t workspace_bytes,
                                void* stream) {
  if (B < 1 || Hq < 1 || Hkv < 1 || S < 1 || a < 0 || n < 1) return SEP_EINVAL;
  if (Hq % Hkv != 0 || B > 65535 || Hq > 65535) return SEP_EINVAL;
  if (dtype != SEP_F32 && dtype != SEP_BF16) return SEP_EDTYPE;
  if (dtype == SEP_BF16 && D != 64 && D != 128) return SEP_EDTYPE;
  if (dtype == SEP_F32 && D != 32 && D != 64 && D != 128) return SEP_EDTYPE;
  if (!q || !k || !v || !is_sep || !prefix || !idx || !out || !workspace) return SEP_ENULL;
  if (!sep::aligned16(q) || !sep::aligned16(k) || !sep::aligned16(v) || !sep::aligned16(out))
    return SEP_EALIGN;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SEP_EALIGN;
  if (workspace_bytes < sep_attn_prefill_workspace(B, Hq, Hkv, S, D, dtype)) return SEP_EINVAL;
  const float sc = scale > 0.f ? scale : 1.f / sqrtf(static_cast<float>(D));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SEP_F32)
    return sep::prefill_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                            static_cast<const float*>(v), prefix, idx, B, Hq, Hkv, S, D, a, n, sc,
                            static_cast<float*>(out), lse, st);
  return sep::prefill_tc(q, k, v, is_sep, prefix, idx, B, Hq, Hkv, S, D, a, n, sc, out, lse,
                         workspace, st);
}
