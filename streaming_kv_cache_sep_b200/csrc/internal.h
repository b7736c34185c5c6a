// Entry points shared between the library's translation units.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sepattn.h"

namespace sep {
int prefill_f32(const float* q, const float* k, const float* v, const int32_t* prefix,
                const int32_t* idx, int B, int Hq, int Hkv, int S, int D, int a, int n,
                float scale, float* out, float* lse, cudaStream_t st);
size_t prefill_tc_workspace(int B, int Hkv, int S, int D);
int prefill_tc(const void* q, const void* k, const void* v, const uint8_t* is_sep,
               const int32_t* prefix, const int32_t* idx, int B, int Hq, int Hkv, int S, int D,
               int a, int n, float scale, void* out, float* lse, void* workspace, cudaStream_t st);
// Run the cache state machine for one token of every sequence (layer-0 part
// of sepcache_append); defined in sepcache.cu.
int cache_advance(const sepcache* c, const uint8_t* is_sep_new, cudaStream_t st);
bool cache_valid(const sepcache* c);
constexpr int kCachePlanHdr = 8;  // plan header words per sequence (see sepcache.cu)
// Tensor map of a bf16 [rows, D] row-major array (D = 64 or 128): tiles of
// 64 columns x box_rows rows, 128-byte swizzled.  Defined in prefill_tc.cu.
bool make_rows_map(CUtensorMap* m, const void* base, int64_t rows, int D, int box_rows);
}  // namespace sep
