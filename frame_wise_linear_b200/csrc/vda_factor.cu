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
// R >= C, of the lower triangle in registers (136 blocks for d = 128).  Pivots
// go in pairs: the owners publish columns k and k + 1 (double-buffered), one
// barrier per pair, and every thread derives the second pivot's column from
// the two published ones.  A non-positive or non-finite pivot sets the
// NOT_SPD bit.
#include "vda_sweep.cuh"

namespace vda {
namespace {

constexpr int kThreads = 160;

template <int D>
__global__ void __launch_bounds__(kThreads, 3) factor_sweep_kernel(float* __restrict__ Mreg, float lam,
                                                                   unsigned* __restrict__ err) {
  // xs[b][0] = column k, xs[b][1] = column k + 1, both before the pair of pivots.
  __shared__ __align__(16) float xs[2][2][D];
  __shared__ __align__(16) float sc[2][4];

  int R, C;
  const bool active = sweep::block_of<D>(threadIdx.x, R, C);
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
  const bool bad = sweep::invert<D>(a, R, C, active, xs, sc, [] { __syncthreads(); });
  if (bad) atomicOr(err, kDevErrNotSpd);
  if (!active) return;

  // a holds -A^{-1}; M = lambda A^{-1} = -lambda a.
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) a[r][c] *= -lam;

  sweep::store_f32<D>(a, R, C, A);
}

template <int D>
cudaError_t launch_d(const vda_problem& p, float* M, unsigned* err, cudaStream_t st) {
  const unsigned slots = (unsigned)(p.B * p.H * (p.T + 1));
  factor_sweep_kernel<D><<<slots, kThreads, 0, st>>>(M, p.lambda, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_factor(const vda_problem& p, float* M, unsigned* err, cudaStream_t st) {
  switch (p.d_k) {
    case 16: return launch_d<16>(p, M, err, st);
    case 32: return launch_d<32>(p, M, err, st);
    case 48: return launch_d<48>(p, M, err, st);
    case 64: return launch_d<64>(p, M, err, st);
    case 80: return launch_d<80>(p, M, err, st);
    case 96: return launch_d<96>(p, M, err, st);
    case 112: return launch_d<112>(p, M, err, st);
    case 128: return launch_d<128>(p, M, err, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace vda
