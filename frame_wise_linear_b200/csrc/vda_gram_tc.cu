// Gram / cross products of the frame-wise joint solve on tcgen05 tensor cores.
//
// For every slot (b, h, t) -- t = 0 is the text, t = 1..T the frames -- this
// computes the normal-equation matrices of "VDN-MiniMax-H3" (aiezz.com),
// section 03, Video Delta Attention item:
//     A_t = K_t^T K_t + lambda I,    B_t = K_t^T V_t        (float32)
// as one MMA chain D = K_t^T [K_t | V_t] with M = 128 (features of K), N = 256
// (features of K then of V), K-dim = tokens.  Inputs are bfloat16, d = 128.
//
// Design (persistent, one CTA per SM, 6 warps):
//   warp 0      TMA producer: 64-token chunks of K_t and V_t, each as two
//               64-feature boxes with the 128-byte swizzle, into a 6-stage ring
//               (32 KB per stage).  Rows past the frame's end read as zeros.
//   warp 1      allocates TMEM (2 x 256 columns) and issues the MMAs from one
//               thread: both operands are MN-major in shared memory (features
//               contiguous), 4 MMAs (16 tokens each) per chunk.
//   warps 2..5  epilogue: TMEM -> registers -> A (+ lambda on the diagonal)
//               and B rows in global memory, while the MMAs of the next slot
//               run into the other TMEM buffer.
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down (waiting, bounded, for its own copies).
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kStages = 6;
constexpr int kChunk = 64;                    // tokens per stage
constexpr int kBox = 64 * 64 * 2;             // one 64 x 64 bf16 box: 8 KB
constexpr int kStageBytes = 4 * kBox;         // K lo/hi features, V lo/hi features
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, /*a MN*/ true, /*b MN*/ true);

struct GramTcParams {
  CUtensorMap mK, mV, mKt, mVt;
  float* A;
  float* Bm;
  unsigned* err;
  int BH, T, n, n_txt;
  float lam;
};

struct Shared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(Shared& sh) { return *reinterpret_cast<volatile int*>(&sh.abort) != 0; }
__device__ __forceinline__ void set_abort(Shared& sh, unsigned* err) {
  atomicOr(err, kDevErrTimeout);
  *reinterpret_cast<volatile int*>(&sh.abort) = 1;
}

__device__ __forceinline__ void slot_info(const GramTcParams& p, int s, int& rows, int& z, bool& text) {
  const int bh = s / (p.T + 1);
  const int t = s % (p.T + 1);
  text = (t == 0);
  rows = text ? p.n_txt : p.n;
  z = text ? bh : bh * p.T + (t - 1);
}

__global__ void __launch_bounds__(kThreads, 1) gram_tc_kernel(const __grid_constant__ GramTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  Shared& sh = *reinterpret_cast<Shared*>(base + kStages * kStageBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int slots = p.BH * (p.T + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.tfull[i], 1);
      mbar_init(&sh.tempty[i], 128);
    }
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.mK);
    tma_prefetch_desc(&p.mV);
    if (p.n_txt > 0) {
      tma_prefetch_desc(&p.mKt);
      tma_prefetch_desc(&p.mVt);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      for (int s = blockIdx.x; s < slots && !aborted(sh); s += gridDim.x) {
        int rows, z;
        bool text;
        slot_info(p, s, rows, z, text);
        const CUtensorMap* mk = text ? &p.mKt : &p.mK;
        const CUtensorMap* mv = text ? &p.mVt : &p.mV;
        for (int r0 = 0; r0 < rows; r0 += kChunk) {
          if (!mbar_wait(&sh.empty[stage], phase ^ 1)) {
            set_abort(sh, p.err);
            break;
          }
          uint8_t* st = stages + stage * kStageBytes;
          mbar_expect_tx(&sh.full[stage], kStageBytes);
          tma_load_3d(st + 0 * kBox, mk, &sh.full[stage], 0, r0, z, pol);
          tma_load_3d(st + 1 * kBox, mk, &sh.full[stage], 64, r0, z, pol);
          tma_load_3d(st + 2 * kBox, mv, &sh.full[stage], 0, r0, z, pol);
          tma_load_3d(st + 3 * kBox, mv, &sh.full[stage], 64, r0, z, pol);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (aborted(sh)) {
        // Error path: wait (bounded) until the chunks that may still be in
        // flight (the last kStages issued) have landed, so no copy is still
        // writing this CTA's shared memory when it exits.
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c) {
          const int st_i = c % kStages;
          const uint32_t ph = (c / kStages) & 1;
          mbar_wait(&sh.full[st_i], ph);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int tb = 0;
      uint32_t tphase = 0;
      const uint32_t sbase = smem_u32(stages);
      for (int s = blockIdx.x; s < slots && !aborted(sh); s += gridDim.x) {
        int rows, z;
        bool text;
        slot_info(p, s, rows, z, text);
        if (rows == 0) continue;
        if (!mbar_wait(&sh.tempty[tb], tphase ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + tb * 256;
        bool first = true;
        for (int r0 = 0; r0 < rows; r0 += kChunk) {
          if (!mbar_wait(&sh.full[stage], phase)) {
            set_abort(sh, p.err);
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * kStageBytes;
#pragma unroll
          for (int k = 0; k < kChunk / 16; ++k) {
            // 16 tokens = 16 rows of 128 bytes; MN blocks of 64 features 8 KB apart.
            const uint64_t desc = smem_desc(sa + k * 16 * 128, kBox, 1024, kSwizzle128B);
            mma_bf16_ss(d, desc, desc, kIdesc, first ? 0u : 1u);
            first = false;
          }
          mma_commit(&sh.empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted(sh)) break;
        mma_commit(&sh.tfull[tb]);
        tb ^= 1;
        if (tb == 0) tphase ^= 1;
      }
      // Make sure no MMA is still running before TMEM is released.
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp % 4;            // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;     // feature index i of D
    int tb = 0;
    uint32_t tphase = 0;
    for (int s = blockIdx.x; s < slots; s += gridDim.x) {
      int rows, z;
      bool text;
      slot_info(p, s, rows, z, text);
      float* Ar = p.A + (size_t)s * 128 * 128 + (size_t)row * 128;
      float* Br = p.Bm + (size_t)s * 128 * 128 + (size_t)row * 128;
      if (rows == 0) {  // no tokens: A = lambda I, B = 0
        for (int c = 0; c < 128; c += 4) {
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
          if (row >= c && row < c + 4) (&a.x)[row - c] = p.lam;
          *reinterpret_cast<float4*>(Ar + c) = a;
          *reinterpret_cast<float4*>(Br + c) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      // Keep the warp converged: tcgen05.ld below is a warp-wide instruction.
      if (__any_sync(0xffffffffu, aborted(sh))) break;
      const bool ok = mbar_wait(&sh.tfull[tb], tphase);
      if (!__all_sync(0xffffffffu, ok)) {
        set_abort(sh, p.err);
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem + tb * 256 + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int chunk = 0; chunk < 8; ++chunk) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + chunk * 32, r);
        tmem_ld_wait();
        float* dst = chunk < 4 ? Ar + chunk * 32 : Br + (chunk - 4) * 32;
        const int col0 = chunk * 32;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          float4 v = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]), __uint_as_float(r[j + 2]),
                                 __uint_as_float(r[j + 3]));
          if (chunk < 4 && row >= col0 + j && row < col0 + j + 4) (&v.x)[row - col0 - j] += p.lam;
          *reinterpret_cast<float4*>(dst + j) = v;
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.tempty[tb]);
      tb ^= 1;
      if (tb == 0) tphase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gram_tc(const vda_problem& p, const __nv_bfloat16* K, const __nv_bfloat16* V,
                           const __nv_bfloat16* Kt, const __nv_bfloat16* Vt, float* A, float* Bm,
                           unsigned* err, cudaStream_t st) {
  GramTcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int BH = p.B * p.H;
  if (!make_bf16_rows_map(&prm.mK, K, p.n, BH * p.T, 64) || !make_bf16_rows_map(&prm.mV, V, p.n, BH * p.T, 64))
    return cudaErrorInvalidValue;
  if (p.n_txt > 0 && (!make_bf16_rows_map(&prm.mKt, Kt, p.n_txt, BH, 64) || !make_bf16_rows_map(&prm.mVt, Vt, p.n_txt, BH, 64)))
    return cudaErrorInvalidValue;
  prm.A = A;
  prm.Bm = Bm;
  prm.err = err;
  prm.BH = BH;
  prm.T = p.T;
  prm.n = p.n;
  prm.n_txt = p.n_txt;
  prm.lam = p.lambda;
  const size_t smem = 1024 + kStages * kStageBytes + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int slots = BH * (p.T + 1);
  const int grid = slots < sms ? slots : sms;
  gram_tc_kernel<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
