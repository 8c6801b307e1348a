// The symmetric sweep operator on a d x d SPD matrix held as 8x8 register
// blocks of its lower triangle (one block per thread): the factor step of the
// float32 path.
//
// Sweeping pivot k maps a_kk -> -1/a_kk, a_ik -> a_ik/a_kk and
// a_ij -> a_ij - a_ik a_kj / a_kk (in-place Gauss-Jordan with diagonal pivots,
// which are the positive LDL^T pivots of an SPD matrix); after all pivots the
// matrix is -A^{-1}.  Each pivot is one symmetric rank-1 update: with
// x = column k (x_k := -1), p = 1/a_kk and row/column k zeroed, a -= x (p x)^T.
// Pivots go in pairs: the owners publish columns k and k + 1 and the pair's
// scalars, one barrier per pair, and every thread derives the second pivot's
// column from the two.
#pragma once

#include "vda_internal.cuh"

namespace vda {
namespace sweep {

// Block (R, C), R >= C, of the lower triangle owned by thread `tid` (blocks
// enumerated row by row); false for threads past the last block.
template <int D>
__device__ __forceinline__ bool block_of(int tid, int& R, int& C) {
  constexpr int NB = D / 8;
  R = C = 0;
  if (tid >= NB * (NB + 1) / 2) return false;
  int r = 0;
  while ((r + 1) * (r + 2) / 2 <= tid) ++r;
  R = r;
  C = tid - r * (r + 1) / 2;
  return true;
}

// Runs all D pivots on `a` (this thread's block).  `xs` is shared scratch of
// [2][2][D] floats and `sc` of [2][4] floats (16-byte aligned); `sync` is a
// barrier over all threads taking part (inactive ones included).  Returns
// true if a pivot was not positive and finite.  On return a holds this block
// of -A^{-1}.
//
// Each pivot is applied without zeroing its row and column: with
// x = column k except x_k = a_kk - 1 and p = 1/a_kk, the update
// a -= x (p x)^T leaves exactly the swept row and column k, and the swept
// diagonal entry after subtracting a further 2.  For the second pivot of a
// pair, column k + 1 after the first is v - x g with g = p u_{k+1}.
template <int D, typename Sync>
__device__ __forceinline__ bool invert(float (&a)[8][8], int R, int C, bool active, float (*xs)[2][D],
                                       float (*sc)[4], Sync sync) {
  constexpr int NB = D / 8;
  bool bad = false;

  // Publishes columns k and k + 1 = 8K + kk, 8K + kk + 1 (current values) into
  // buffer b; the owner of the diagonal block also publishes the pair's
  // scalars p1 = 1/a_kk, g = p1 a_{k+1,k} and p2 = 1/(a_{k+1,k+1} - a_{k+1,k} g).
  auto publish = [&](int K, auto kk_c, int b) {
    constexpr int kk = decltype(kk_c)::value;
    if (!active) return;
    if (C == K) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        xs[b][0][8 * R + r] = a[r][kk];
        xs[b][1][8 * R + r] = a[r][kk + 1];
      }
    }
    if (R == K && C < K) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        xs[b][0][8 * C + c] = a[kk][c];
        xs[b][1][8 * C + c] = a[kk + 1][c];
      }
    }
    if (R == K && C == K) {
      const float uk = a[kk][kk], uk1 = a[kk + 1][kk], vk1 = a[kk + 1][kk + 1];
      const float p1 = 1.f / uk;
      const float g = p1 * uk1;
      const float piv2 = vk1 - uk1 * g;
      if (!(uk > 0.f) || !isfinite(uk) || !(piv2 > 0.f) || !isfinite(piv2)) bad = true;
      sc[b][0] = p1;
      sc[b][1] = g;
      sc[b][2] = 1.f / piv2;
    }
  };
  auto load8 = [&](const float* src, float (&v)[8]) {
    const float4 lo = *reinterpret_cast<const float4*>(src);
    const float4 hi = *reinterpret_cast<const float4*>(src + 4);
    v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
    v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
  };

  publish(0, std::integral_constant<int, 0>{}, 0);
  int buf = 0;
#pragma unroll 1
  for (int K = 0; K < NB; ++K) {
    auto pair = [&](auto kk_c) {
      constexpr int kk = decltype(kk_c)::value;
      sync();
      if (active) {
        const float4 s4 = *reinterpret_cast<const float4*>(sc[buf]);
        const float p1 = s4.x, g = s4.y, p2 = s4.z;
        const bool rk = (R == K), ck = (C == K);
        float xr[8], xc[8], yc[8];
        load8(&xs[buf][0][8 * R], xr);
        load8(&xs[buf][0][8 * C], xc);
        if (rk) xr[kk] -= 1.f;
        if (ck) xc[kk] -= 1.f;
        // ---- pivot k
#pragma unroll
        for (int i = 0; i < 8; ++i) yc[i] = p1 * xc[i];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) a[r][c] = fmaf(-xr[r], yc[c], a[r][c]);
        if (rk && ck) a[kk][kk] -= 2.f;
        // ---- pivot k + 1: x' = v - x g, x'_{k+1} -= 1
        float vr[8], vc[8];
        load8(&xs[buf][1][8 * R], vr);
        load8(&xs[buf][1][8 * C], vc);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          vr[i] = fmaf(-xr[i], g, vr[i]);
          vc[i] = fmaf(-xc[i], g, vc[i]);
        }
        if (rk) vr[kk + 1] -= 1.f;
        if (ck) vc[kk + 1] -= 1.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) yc[i] = p2 * vc[i];
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) a[r][c] = fmaf(-vr[r], yc[c], a[r][c]);
        if (rk && ck) a[kk + 1][kk + 1] -= 2.f;
      }
      buf ^= 1;
      if constexpr (kk + 2 < 8) {
        publish(K, std::integral_constant<int, kk + 2>{}, buf);
      } else {
        if (K + 1 < NB) publish(K + 1, std::integral_constant<int, 0>{}, buf);
      }
    };
    pair(std::integral_constant<int, 0>{});
    pair(std::integral_constant<int, 2>{});
    pair(std::integral_constant<int, 4>{});
    pair(std::integral_constant<int, 6>{});
  }
  return bad;
}

// Writes this thread's block and its transpose into a row-major D x D matrix.
template <int D>
__device__ __forceinline__ void store_f32(const float (&a)[8][8], int R, int C, float* A) {
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    float* row = A + (size_t)(8 * R + r) * D + 8 * C;
    *reinterpret_cast<float4*>(row) = make_float4(a[r][0], a[r][1], a[r][2], a[r][3]);
    *reinterpret_cast<float4*>(row + 4) = make_float4(a[r][4], a[r][5], a[r][6], a[r][7]);
  }
  if (R != C) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float* row = A + (size_t)(8 * C + c) * D + 8 * R;
      *reinterpret_cast<float4*>(row) = make_float4(a[0][c], a[1][c], a[2][c], a[3][c]);
      *reinterpret_cast<float4*>(row + 4) = make_float4(a[4][c], a[5][c], a[6][c], a[7][c]);
    }
  }
}

}  // namespace sweep
}  // namespace vda
