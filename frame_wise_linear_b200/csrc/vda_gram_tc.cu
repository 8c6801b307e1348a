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
//               64-feature boxes with the 128-byte swizzle, into a 5-stage ring
//               (32 KB per stage).  Rows past the frame's end read as zeros.
//   warp 1      allocates TMEM (2 x 256 columns) and issues the MMAs from one
//               thread: both operands are MN-major in shared memory (features
//               contiguous), 4 MMAs (16 tokens each) per chunk.
//   warps 2..5  epilogue: TMEM -> registers -> 32-column chunks of A (+ lambda
//               on the diagonal) and B, staged swizzled in shared memory and
//               written by TMA stores, while the MMAs of the next slot run into
//               the other TMEM buffer.
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down (waiting, bounded, for its own copies).
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kStages = 5;
constexpr int kChunk = 64;                    // tokens per stage
constexpr int kBox = 64 * 64 * 2;             // one 64 x 64 bf16 box: 8 KB
constexpr int kStageBytes = 4 * kBox;         // K lo/hi features, V lo/hi features
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;           // two 256-column accumulators
constexpr int kOutChunk = 128 * 32 * 4;       // epilogue staging: 32 float32 columns x 128 rows
constexpr int kEpiBar = 1;                    // named barrier of the 4 epilogue warps
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 256, /*a MN*/ true, /*b MN*/ true);

struct GramTcParams {
  CUtensorMap mK, mV, mKt, mVt;
  CUtensorMap mA, mB;   // [slots * 128][128] float32, 32 x 128 boxes
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
  uint8_t* ostage = base + kStages * kStageBytes;   // 2 x output staging chunk
  Shared& sh = *reinterpret_cast<Shared*>(ostage + 2 * kOutChunk);

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
    // D row by row (lane = feature i) into swizzled 32-column staging chunks,
    // each stored by one TMA store: chunks 0..3 are A (+ lambda on the
    // diagonal), 4..7 are B.
    const int quarter = warp % 4;            // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;     // feature index i of D
    const bool leader = (warp == 2 && lane == 0);
    int tb = 0, nst = 0;
    uint32_t tphase = 0;
    for (int s = blockIdx.x; s < slots; s += gridDim.x) {
      int rows, z;
      bool text;
      slot_info(p, s, rows, z, text);
      if (__any_sync(0xffffffffu, aborted(sh))) break;
      if (rows > 0) {
        const bool ok = mbar_wait(&sh.tfull[tb], tphase);
        if (!__all_sync(0xffffffffu, ok)) {
          set_abort(sh, p.err);
          break;
        }
        tc_fence_after();
      }
      const uint32_t taddr = tmem + tb * 256 + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int chunk = 0; chunk < 8; ++chunk) {
        uint32_t r[32];
        if (rows > 0) {
          tmem_ld_32x32b_x32(taddr + chunk * 32, r);
          tmem_ld_wait();
        } else {  // no tokens: A = lambda I, B = 0
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0u;
        }
        if (chunk < 4) {
          const int j = row - chunk * 32;   // the diagonal entry, if in this chunk
#pragma unroll
          for (int jj = 0; jj < 32; ++jj)
            if (jj == j) r[jj] = __float_as_uint(__uint_as_float(r[jj]) + p.lam);
        }
        uint8_t* stg = ostage + (nst & 1) * kOutChunk;
        if (leader) bulk_wait_read<1>();      // the store two chunks back has read this buffer
        named_bar_sync(kEpiBar, 128);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + sw128(row, q)) = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        fence_proxy_async_smem();
        named_bar_sync(kEpiBar, 128);
        if (leader) {
          tma_store_2d(chunk < 4 ? &p.mA : &p.mB, stg, (chunk % 4) * 32, s * 128);
          bulk_commit();
        }
        ++nst;
      }
      if (rows > 0) {
        tc_fence_before();
        mbar_arrive(&sh.tempty[tb]);
        tb ^= 1;
        if (tb == 0) tphase ^= 1;
      }
    }
    if (leader) bulk_wait<0>();               // A and B stores complete before exit
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
  const long long rows = (long long)BH * (p.T + 1) * 128;
  if (!make_f32_rows_map(&prm.mA, A, rows, 128) || !make_f32_rows_map(&prm.mB, Bm, rows, 128))
    return cudaErrorInvalidValue;
  prm.A = A;
  prm.Bm = Bm;
  prm.err = err;
  prm.BH = BH;
  prm.T = p.T;
  prm.n = p.n;
  prm.n_txt = p.n_txt;
  prm.lam = p.lambda;
  const size_t smem = 1024 + kStages * kStageBytes + 2 * kOutChunk + sizeof(Shared);
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
