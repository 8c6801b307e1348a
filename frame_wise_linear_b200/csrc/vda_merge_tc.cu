// The branch merge of the hybrid attention on tcgen05 tensor cores: each
// branch's gated output through its own output projection, summed.
//
// "VDN-MiniMax-H3" (aiezz.com), section 03, gate fusion item (restated in the
// laicaila.com page, section 技术原理): the two branches' outputs have
// different scales, so each has its own content-dependent sigmoid gate and
// its own output projection before they are merged.  With the gates applied
// by the branches themselves (the VDA readout applies the linear branch's),
// the merge is one product over the two branches' concatenated features:
//     Y = O_lin W_lin + O_sm W_sm = [O_lin | O_sm] [W_lin ; W_sm]
// O_lin, O_sm: [tokens, K] bf16 (heads concatenated, the token-major layout
// of the attention outputs); W_lin, W_sm: [K, D] bf16; Y: [tokens, D] bf16,
// float32 accumulation.  O_sm may be absent (Y = O_lin W_lin).
//
// Design (persistent, one CTA per SM, 6 warps), output tiles of 128 tokens x
// 256 columns, N-tiles of one M-tile on neighbouring CTAs so the A rows are
// shared in L2:
//   warp 0     TMA producer: per 64-feature K block, the A box (128 rows x 64
//              features, K-major) and four W boxes (64 K rows x 64 columns,
//              MN-major), through a 4-stage ring of 48 KB.
//   warp 1     TMEM (two 256-column accumulators) and the MMAs (M = 128,
//              N = 256, K = 16; four per K block), the branches one after the
//              other into the same accumulator.
//   warps 2..5 epilogue: TMEM -> bf16 -> a 64-column staging box (two, used
//              in turn) -> TMA store; the tile's accumulator is free as soon
//              as its last columns are in registers.
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;       // 16 KB
constexpr int kWBox = kBK * 64 * 2;          // 64 K rows x 64 columns: 8 KB
constexpr int kBBytes = kBN / 64 * kWBox;    // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kStgBytes = kBM * 64 * 2;      // one 64-column output box: 16 KB
constexpr int kEpiBar = 1;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, /*a MN*/ false, /*b MN*/ true);

struct MergeParams {
  CUtensorMap mA0, mA1;    // O_lin, O_sm: [tokens][K], 64 x 128 boxes
  CUtensorMap mW0, mW1;    // W_lin, W_sm: [K][D], 64 x 64 boxes
  CUtensorMap mY;          // [tokens][D], 64 x 128 boxes
  unsigned* err;
  int m_tiles, n_tiles;
  int kb0, kb;             // K blocks of the linear branch; of both
  int stall;               // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t full[kStages], empty[kStages];
  uint64_t t_full[2], t_empty[2];
  uint64_t drain;
  uint64_t never;          // testing hook: nothing arrives on it
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool aborted(Shared& sh) { return *reinterpret_cast<volatile int*>(&sh.abort) != 0; }
__device__ __forceinline__ void set_abort(Shared& sh, unsigned* err) {
  atomicOr(err, kDevErrTimeout);
  *reinterpret_cast<volatile int*>(&sh.abort) = 1;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreads, 1) merge_tc_kernel(const __grid_constant__ MergeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;
  uint8_t* stg = base + kStages * kStageBytes;
  Shared& sh = *reinterpret_cast<Shared*>(stg + 2 * kStgBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int tiles = p.m_tiles * p.n_tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.t_full[i], 1);
      mbar_init(&sh.t_empty[i], 128);
    }
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.never, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.mA0);
    tma_prefetch_desc(&p.mW0);
    tma_prefetch_desc(&p.mY);
    if (p.kb > p.kb0) {
      tma_prefetch_desc(&p.mA1);
      tma_prefetch_desc(&p.mW1);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_a = policy_evict_last();   // A rows serve the M-tile's N-tiles
      const uint64_t pol_w = policy_evict_last();   // W serves every M-tile
      int it = 0, issued = 0;
      for (int t = blockIdx.x; t < tiles && !aborted(sh); t += gridDim.x) {
        const int m0 = (t / p.n_tiles) * kBM, n0 = (t % p.n_tiles) * kBN;
        for (int kb = 0; kb < p.kb; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&sh.empty[s], ((it / kStages) & 1) ^ 1)) {
            set_abort(sh, p.err);
            break;
          }
          const bool lin = kb < p.kb0;
          const int k0 = (lin ? kb : kb - p.kb0) * kBK;
          uint8_t* st = ring + s * kStageBytes;
          mbar_expect_tx(&sh.full[s], kStageBytes);
          tma_load_2d(st, lin ? &p.mA0 : &p.mA1, &sh.full[s], k0, m0, pol_a);
#pragma unroll
          for (int j = 0; j < kBN / 64; ++j)
            tma_load_2d(st + kABytes + j * kWBox, lin ? &p.mW0 : &p.mW1, &sh.full[s], n0 + 64 * j, k0, pol_w);
          ++issued;
        }
      }
      if (aborted(sh))   // the loads still in flight land before exit
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
          mbar_wait(&sh.full[c % kStages], (c / kStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      int it = 0, i = 0;
      const uint64_t d0 = smem_desc(smem_u32(ring), 16, 1024, kSwizzle128B);
      for (int t = blockIdx.x; t < tiles && ok; t += gridDim.x, ++i) {
        const int tb = i & 1;
        if (!(ok = !aborted(sh) && mbar_wait(&sh.t_empty[tb], ((i >> 1) & 1) ^ 1))) break;
        tc_fence_after();
        const uint32_t d = tmem + tb * kBN;
        for (int kb = 0; kb < p.kb; ++kb, ++it) {
          const int s = it % kStages;
          const bool stall = p.stall == VDA_TEST_STALL_MERGE && blockIdx.x == 0 && it == 0;
          if (!(ok = mbar_wait_or_stall(&sh.full[s], (it / kStages) & 1, &sh.never, stall))) break;
          tc_fence_after();
          const uint32_t so = s * kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major, 16 features = 32 bytes in the 128-byte row; B: MN-major,
            // 16 K rows of 128 bytes, 64-column blocks one W box apart.
            const uint64_t a = d0 + ((so + kk * 32) >> 4);
            uint64_t b = smem_desc(smem_u32(ring + so + kABytes + kk * 16 * 128), kWBox, 1024, kSwizzle128B);
            mma_bf16_ss(d, a, b, kIdesc, (kb | kk) ? 1u : 0u);
          }
          mma_commit(&sh.empty[s]);
        }
        if (!ok) break;
        mma_commit(&sh.t_full[tb]);
      }
      if (!ok) set_abort(sh, p.err);
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    const int row = (warp % 4) * 32 + lane;   // tile row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    int i = 0, nst = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++i) {
      const int tb = i & 1;
      const int m0 = (t / p.n_tiles) * kBM, n0 = (t % p.n_tiles) * kBN;
      bool ok = !aborted(sh) && mbar_wait(&sh.t_full[tb], (i >> 1) & 1);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(kEpiBar, 128, !ok)) break;   // one decision for the four warps
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < kBN / 64; ++c, ++nst) {
        uint8_t* box = stg + (nst & 1) * kStgBytes;
        if (leader) bulk_wait_read<1>();      // the store two boxes back has read this buffer
        named_bar_sync(kEpiBar, 128);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + tb * kBN + lane_off + c * 64 + h * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(box + sw128(row, h * 4 + q)) =
                make_uint4(pack_bf16(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                           pack_bf16(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                           pack_bf16(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                           pack_bf16(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
        }
        if (c == kBN / 64 - 1) {              // the accumulator is in registers: free it
          tc_fence_before();
          mbar_arrive(&sh.t_empty[tb]);
        }
        fence_proxy_async_smem();
        named_bar_sync(kEpiBar, 128);
        if (leader) {                         // columns and rows past Y's edge are clipped
          tma_store_2d(&p.mY, box, n0 + 64 * c, m0);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_merge_tc(long long tokens, int K, int D, const __nv_bfloat16* O_lin, const __nv_bfloat16* W_lin,
                            const __nv_bfloat16* O_sm, const __nv_bfloat16* W_sm, __nv_bfloat16* Y, unsigned* err,
                            cudaStream_t st, int stall) {
  MergeParams prm;
  memset(&prm, 0, sizeof(prm));
  if (!make_bf16_2d_map(&prm.mA0, O_lin, tokens, K, 64, kBM) || !make_bf16_2d_map(&prm.mW0, W_lin, K, D, 64, kBK) ||
      !make_bf16_2d_map(&prm.mY, Y, tokens, D, 64, kBM))
    return cudaErrorInvalidValue;
  const bool two = O_sm != nullptr;
  if (two && (!make_bf16_2d_map(&prm.mA1, O_sm, tokens, K, 64, kBM) ||
              !make_bf16_2d_map(&prm.mW1, W_sm, K, D, 64, kBK)))
    return cudaErrorInvalidValue;
  prm.err = err;
  prm.stall = stall;
  prm.m_tiles = (int)((tokens + kBM - 1) / kBM);
  prm.n_tiles = (D + kBN - 1) / kBN;
  prm.kb0 = K / kBK;
  prm.kb = two ? 2 * prm.kb0 : prm.kb0;
  const size_t smem = 1024 + kStages * kStageBytes + 2 * kStgBytes + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(merge_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)prm.m_tiles * prm.n_tiles;
  const int grid = (int)(tiles < sms ? tiles : sms);
  merge_tc_kernel<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
