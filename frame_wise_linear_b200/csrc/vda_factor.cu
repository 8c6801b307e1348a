// Factor step: M_t = lambda A_t^{-1} for every slot (frames and text).
//
// "VDN-MiniMax-H3" (aiezz.com), section 03, Video Delta Attention item: each
// frame's new state comes from a joint solve of the normal equations
// A_t S = lambda S_{t-1} + B_t.  The scan uses the equivalent form
//     S_t = M_t (S_{t-1} + B_t / lambda),   M_t = lambda A_t^{-1},
// so this step needs only M_t (non-expansive: ||M_t||_2 <= 1).
//
// Method: the symmetric sweep operator (in-place Gauss-Jordan with diagonal
// pivots, which are the positive LDL^T pivots of an SPD matrix).  Sweeping
// pivot k maps
//     a_kk -> -1/a_kk,  a_ik -> a_ik/a_kk,  a_ij -> a_ij - a_ik a_kj / a_kk,
// and after all pivots the matrix is -A^{-1}.  Written as one symmetric
// rank-1 update per pivot: with x = column k (x_k := -1), p = 1/a_kk and
// row/column k zeroed first, a -= x (p x)^T.  n^3/2 FMA on the lower triangle.
//
// Layout: one CTA per slot, 160 threads; thread t owns one 8x8 block (R, C),
// R >= C, of the lower triangle in registers (136 blocks for d = 128).  Per
// pivot, the owners of column k publish it (double-buffered) and one barrier
// separates pivots.  A non-positive or non-finite pivot sets the NOT_SPD bit.
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

constexpr int kThreads = 160;

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Writes 8 consecutive k-values of row m of M as bf16 hi and lo chunks of the
// K-major, 128-byte-swizzled MMA operand image (two 64-column halves of 16 KB).
__device__ __forceinline__ void store_split_chunk(uint8_t* hi, uint8_t* lo, int m, int kchunk, const float (&v)[8]) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h[i] = __bfloat162float(__float2bfloat16_rn(v[i]));
    l[i] = v[i] - h[i];
  }
  const uint32_t off = (kchunk / 8) * 16384u + sm100::sw128(m, kchunk % 8);
  *reinterpret_cast<uint4*>(hi + off) = make_uint4(pack2(h[0], h[1]), pack2(h[2], h[3]), pack2(h[4], h[5]), pack2(h[6], h[7]));
  *reinterpret_cast<uint4*>(lo + off) = make_uint4(pack2(l[0], l[1]), pack2(l[2], l[3]), pack2(l[4], l[5]), pack2(l[6], l[7]));
}

template <int D, bool kSplitOut>
__global__ void __launch_bounds__(kThreads) factor_sweep_kernel(float* __restrict__ Mreg, float lam,
                                                                unsigned* __restrict__ err) {
  constexpr int NB = D / 8;
  constexpr int NBLK = NB * (NB + 1) / 2;
  __shared__ float xs[2][D];
  __shared__ float pinv[2];

  const int tid = threadIdx.x;
  const bool active = tid < NBLK;
  // block (R, C) of the lower triangle, enumerated row by row
  int R = 0, C = 0;
  if (active) {
    int r = 0;
    while ((r + 1) * (r + 2) / 2 <= tid) ++r;
    R = r;
    C = tid - r * (r + 1) / 2;
  }
  float* A = Mreg + (size_t)blockIdx.x * D * D;

  float a[8][8];
  if (active) {
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const float4 v0 = *reinterpret_cast<const float4*>(A + (size_t)(8 * R + r) * D + 8 * C);
      const float4 v1 = *reinterpret_cast<const float4*>(A + (size_t)(8 * R + r) * D + 8 * C + 4);
      a[r][0] = v0.x; a[r][1] = v0.y; a[r][2] = v0.z; a[r][3] = v0.w;
      a[r][4] = v1.x; a[r][5] = v1.y; a[r][6] = v1.z; a[r][7] = v1.w;
    }
  }
  bool bad = false;

  // Publishes column k (pre-update values of the next pivot) into buffer b.
  auto publish = [&](int K, auto kk_c, int b) {
    constexpr int kk = decltype(kk_c)::value;
    if (!active) return;
    if (C == K) {
#pragma unroll
      for (int r = 0; r < 8; ++r) xs[b][8 * R + r] = a[r][kk];
    }
    if (R == K && C < K) {
#pragma unroll
      for (int c = 0; c < 8; ++c) xs[b][8 * C + c] = a[kk][c];
    }
    if (R == K && C == K) {
      const float piv = a[kk][kk];
      if (!(piv > 0.f) || !isfinite(piv)) bad = true;
      pinv[b] = 1.f / piv;
      xs[b][8 * K + kk] = -1.f;
    }
  };

  publish(0, std::integral_constant<int, 0>{}, 0);
  int buf = 0;
#pragma unroll 1
  for (int K = 0; K < NB; ++K) {
    auto step = [&](auto kk_c) {
      constexpr int kk = decltype(kk_c)::value;
      __syncthreads();
      if (active) {
        const float p = pinv[buf];
        float xr[8], yc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          xr[i] = xs[buf][8 * R + i];
          yc[i] = p * xs[buf][8 * C + i];
        }
        if (R == K) {
#pragma unroll
          for (int c = 0; c < 8; ++c) a[kk][c] = 0.f;
        }
        if (C == K) {
#pragma unroll
          for (int r = 0; r < 8; ++r) a[r][kk] = 0.f;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r)
#pragma unroll
          for (int c = 0; c < 8; ++c) a[r][c] = fmaf(-xr[r], yc[c], a[r][c]);
      }
      buf ^= 1;
      if constexpr (kk < 7) {
        publish(K, std::integral_constant<int, kk + 1>{}, buf);
      } else {
        if (K + 1 < NB) publish(K + 1, std::integral_constant<int, 0>{}, buf);
      }
    };
    step(std::integral_constant<int, 0>{});
    step(std::integral_constant<int, 1>{});
    step(std::integral_constant<int, 2>{});
    step(std::integral_constant<int, 3>{});
    step(std::integral_constant<int, 4>{});
    step(std::integral_constant<int, 5>{});
    step(std::integral_constant<int, 6>{});
    step(std::integral_constant<int, 7>{});
  }
  if (bad) atomicOr(err, kDevErrNotSpd);
  if (!active) return;

  // a holds -A^{-1}; M = lambda A^{-1} = -lambda a.
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) a[r][c] *= -lam;

  if constexpr (kSplitOut) {
    uint8_t* hi = reinterpret_cast<uint8_t*>(A);
    uint8_t* lo = hi + 32768;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float v[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) v[c] = a[r][c];
      store_split_chunk(hi, lo, 8 * R + r, C, v);
    }
    if (R != C) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float v[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) v[r] = a[r][c];
        store_split_chunk(hi, lo, 8 * C + c, R, v);
      }
    }
  } else {
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
}

template <int D, bool kSplit>
cudaError_t launch_d(const vda_problem& p, float* M, unsigned* err, cudaStream_t st) {
  const unsigned slots = (unsigned)(p.B * p.H * (p.T + 1));
  factor_sweep_kernel<D, kSplit><<<slots, kThreads, 0, st>>>(M, p.lambda, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_factor(const vda_problem& p, float* M, unsigned* err, bool split_bf16, cudaStream_t st) {
  if (split_bf16) {
    if (p.d_k != 128) return cudaErrorInvalidValue;
    return launch_d<128, true>(p, M, err, st);
  }
  switch (p.d_k) {
    case 16: return launch_d<16, false>(p, M, err, st);
    case 32: return launch_d<32, false>(p, M, err, st);
    case 48: return launch_d<48, false>(p, M, err, st);
    case 64: return launch_d<64, false>(p, M, err, st);
    case 80: return launch_d<80, false>(p, M, err, st);
    case 96: return launch_d<96, false>(p, M, err, st);
    case 112: return launch_d<112, false>(p, M, err, st);
    case 128: return launch_d<128, false>(p, M, err, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vda
