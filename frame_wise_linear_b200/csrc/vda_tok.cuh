// Token tiles of either input layout, for the tensor-core kernels.  A frame
// unit is u = (b H + h) T + t; a text unit is u = b H + h.  The descriptors
// come from make_tok_map (vda_tma.cu): layout 0 is [B][H][T][n][128], a 3-D
// map (c, r, u); layout 1 is [B][T][n][H][128], a 5-D map (c, h, r, t, b);
// the text has T = 1.  In layout 1 a unit's position is decoded once
// (tok_pos: integer divisions) and reused for all its loads and stores.
#pragma once

#include "sm100.cuh"

namespace vda {

struct TokGeom {
  int layout;   // 0 or 1 (vda_layout)
  int H, T;
};

struct TokPos {
  int unit, t, h, b;   // t, h, b decoded in layout 1 only
};

__device__ __forceinline__ TokPos tok_pos(const TokGeom& g, int unit, bool text) {
  if (g.layout == 0) return TokPos{unit, 0, 0, 0};
  if (text) return TokPos{unit, 0, unit % g.H, unit / g.H};
  const int bh = unit / g.T;
  return TokPos{unit, unit % g.T, bh % g.H, bh / g.H};
}

// Features x .. x + 63 of tokens y .. y + box_rows - 1 of the unit at `q`.
__device__ __forceinline__ void tok_load(void* dst, const CUtensorMap* m, uint64_t* bar, const TokGeom& g,
                                         const TokPos& q, int x, int y, uint64_t pol) {
  if (g.layout == 1)
    sm100::tma_load_5d(dst, m, bar, x, q.h, y, q.t, q.b, pol);
  else
    sm100::tma_load_3d(dst, m, bar, x, y, q.unit, pol);
}

__device__ __forceinline__ void tok_store(const CUtensorMap* m, const void* src, const TokGeom& g, const TokPos& q,
                                          int x, int y) {
  if (g.layout == 1)
    sm100::tma_store_5d(m, src, x, q.h, y, q.t, q.b);
  else
    sm100::tma_store_3d(m, src, x, y, q.unit);
}

// Element offset of token row 0 of the unit at `q` in a tensor with `rows`
// tokens per unit (n, or n_txt for the text), and between consecutive rows.
__device__ __forceinline__ size_t tok_base(const TokGeom& g, const TokPos& q, int rows, bool text) {
  if (g.layout == 0) return (size_t)q.unit * rows * 128;
  const size_t T = text ? 1 : g.T;
  return (((size_t)q.b * T + q.t) * rows * g.H + q.h) * 128;
}
__device__ __forceinline__ size_t tok_row_stride(const TokGeom& g) { return g.layout == 0 ? 128 : (size_t)g.H * 128; }

}  // namespace vda
