// Host construction of the tensor maps the kernels load through.
#pragma once

#include <cuda.h>

#include "pa.h"

namespace pa {

// The cache [NB, bs, Hkv, D] as a 4-D tensor {D, Hkv, bs, NB} (innermost
// first) with box {128 bytes of D, 1, bs, 1}: one 128-byte segment of the K
// (or V) rows of one block for one kv head, 128-byte swizzled.
pa_status make_cache_map(CUtensorMap* m, const void* base, pa_dtype dt, int64_t NB, int bs, int Hkv,
                         int D);

// The same cache as a 4-D tensor {D, bs, Hkv, NB} (tokens before heads; the
// strides keep the memory order) with box {128 bytes of D, bs, hg, 1}: one
// 128-byte segment of the K (or V) rows of one block for hg neighbouring kv
// heads, laid out head-major in shared memory ([head][token][128 B]), so each
// head's rows form the same swizzled tile as a one-head box.
pa_status make_cache_map_heads(CUtensorMap* m, const void* base, pa_dtype dt, int64_t NB, int bs,
                               int Hkv, int D, int hg);

// Token-major rows [T, H, D] as a 3-D tensor {D, H, T} with box
// {128 bytes of D, box_h, box_t}: box_t tokens x box_h heads of one 128-byte
// segment, 128-byte swizzled, rows past T read as zeros.
pa_status make_rows_map(CUtensorMap* m, const void* base, pa_dtype dt, int64_t T, int H, int D,
                        int box_h, int box_t);

}  // namespace pa
