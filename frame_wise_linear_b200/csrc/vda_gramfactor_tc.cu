// Gram / cross products and the factor step in one kernel, on tcgen05 tensor
// cores (bf16 or e4m3 inputs, d = 128).
//
// For every slot (b, h, t) -- t = 0 is the text, t = 1..T the frames -- this
// computes, after "VDN-MiniMax-H3" (aiezz.com), section 03, Video Delta
// Attention item (each frame's state comes from a joint solve of the normal
// equations over all of its tokens):
//     A_t = K_t^T K_t + lambda I,    B_t = K_t^T V_t          (float32)
//     M_t = lambda A_t^{-1}                                   (written as bf16 hi + lo)
// The scan then runs S_t = M_t (S_{t-1} + B_t / lambda).
//
// Gram: per 16 tokens (bf16, kind::f16) or 32 tokens (e4m3, kind::f8f6f4),
// two MMAs into TMEM: A += K^T K and B += K^T V (M = 128 features of K, N =
// 128, K-dim = tokens).  Products of 8-bit floats are exact in the float32
// accumulator.  With e4m3 inputs (per-tensor scales s_k, s_v) the service
// warps scale the chains to the values' units (A by s_k^2, B by s_k s_v)
// before lambda is added and the sweep runs.
// Factor: A_t stays where the chain left it, in TMEM (lane i = row i), and is
// swept there: the sweep operator taken 8 pivots at a time in its Cholesky
// form.  For a pivot block K with P = A_KK = L L^T and X = A[:, K],
//     X~ = X with X~_K = P - I,   Y = X~ L^{-T},   A <- A - Y Y^T,
// leaves the swept block row and column in place; the -2 on the swept
// diagonal commutes with later blocks and is applied once at the end:
// -A^{-1} = A_final - 2I, so M = lambda (2I - A_final).  Each thread forms its
// row of Y; the rank-8 update is three kind::tf32 MMAs (Y hi/lo products above
// float32 rounding, A negated).  A never goes through HBM.
//
// TMEM (512 columns): three 128-column A regions used in turn by successive
// slots, and one 128-column B region.
//
// Design (persistent, one CTA per SM, 14 warps), slots round-robin over CTAs:
//   warp 0      TMA producer: 64-token chunks of K_t and V_t, each as two
//               64-feature boxes with the 128-byte swizzle, 5-stage ring.
//   warp 1      allocates TMEM and issues the Gram MMAs from one thread (both
//               operands MN-major in shared memory), once the slot's A region
//               is free (M of its previous slot written) and B is drained.
//   warps 2..5  service warps, per slot: B_t out (TMEM -> 32-column swizzled
//               chunks -> TMA stores), lambda onto A's diagonal in TMEM, A to
//               the slot's factor group; then M of the previous slot, once
//               its sweep is complete, out of TMEM as bf16 hi/lo in the
//               scan's operand layout, and its A region back to the Gram.
//   warps 6..13 two factor groups of four warps (one thread per row of A),
//               sweeping alternate slots, so that one group's pivot-block
//               work overlaps the other's update MMAs; the first thread of a
//               group issues its update MMAs.
// A non-positive or non-finite pivot sets the NOT_SPD bit; every wait is
// bounded, and a wait that runs out sets the timeout bit and winds the CTA
// down (waiting, bounded, for its own copies and MMAs).
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kStages = 5;
constexpr int kHalfStage = 16384;             // K's part of a stage, then V's
constexpr int kStageBytes = 2 * kHalfStage;
// Per input type: tokens per stage and per MMA.  bf16: 64-token chunks, each
// tensor as two 64-feature boxes (8 KB each), 16 tokens per MMA (kind::f16).
// e4m3: 128-token chunks, each tensor as one 128-feature box (16 KB), 32
// tokens per MMA (kind::f8f6f4).  Both fill a 128-byte-swizzled row per token.
template <bool kF8>
struct GramCfg {
  static constexpr int kChunk = kF8 ? 128 : 64;
  static constexpr int kKTok = kF8 ? 32 : 16;
  static constexpr int kBoxes = kF8 ? 1 : 2;          // boxes per tensor and stage
  static constexpr int kBox = kHalfStage / kBoxes;
};
constexpr int kFacGroups = 2;                 // factor groups, each sweeping its own slot
constexpr int kThreads = 32 * (6 + 4 * kFacGroups);
constexpr int kARegions = 3;                  // TMEM: three 128-column A regions, then B
constexpr uint32_t kBCol = 128 * kARegions;
constexpr uint32_t kTmemCols = 512;
constexpr int kOutChunk = 128 * 32 * 4;       // B staging: 32 float32 columns x 128 rows
constexpr int kEpiBar = 1;                    // named barrier of the B epilogue warps
constexpr int kFacBar0 = 2;                   // named barriers of the factor groups: 2, 3
constexpr int kOp = 128 * 8 * 4;              // factor operand: 128 rows x 8 tf32 (4 KB)
constexpr uint32_t kIdescGram = idesc_bf16_f32(128, 128, /*a MN*/ true, /*b MN*/ true);
constexpr uint32_t kIdescGram8 = idesc_e4m3_f32(128, 128, /*a MN*/ true, /*b MN*/ true);
constexpr uint32_t kIdescUpd = idesc_tf32_f32(128, 128, /*negate A*/ true);

struct GramFactorParams {
  CUtensorMap mK, mV, mKt, mVt;
  CUtensorMap mB;       // [slots * 128][128] float32, 32 x 128 boxes
  uint8_t* M;           // per slot 64 KB: M hi | M lo
  unsigned* err;
  int BH, T, n, n_txt;
  float lam;
  TokGeom g;            // the inputs' layout
  int stall;            // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
  float a_scale;        // e4m3 inputs: A = a_scale K8^T K8 + lambda I, B = b_scale K8^T V8 (1 for bf16)
  float b_scale;
};

struct Shared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t gdone;               // one phase per slot: its Gram chain is complete
  uint64_t bfree;               // one phase per slot: B drained, the B region is free
  uint64_t tempty[kARegions];   // M written: the A region may take the next Gram chain
  uint64_t aready[kFacGroups];  // per group, one phase per slot: lambda on A's diagonal
  uint64_t fin[kFacGroups];     // per group, one phase per slot: sweep complete
  uint64_t upd[kFacGroups];     // per group, one phase per block step
  uint64_t fdone[kFacGroups];   // per group, one phase per slot: all its MMAs complete
  uint64_t drain;
  uint64_t never;               // testing hook: nothing arrives on it
  uint32_t tmem_base;
  int bad;
  int abort;
};

__device__ __forceinline__ bool aborted(Shared& sh) { return *reinterpret_cast<volatile int*>(&sh.abort) != 0; }
__device__ __forceinline__ void set_abort(Shared& sh, unsigned* err) {
  atomicOr(err, kDevErrTimeout);
  *reinterpret_cast<volatile int*>(&sh.abort) = 1;
}

__device__ __forceinline__ void slot_info(const GramFactorParams& p, int s, int& rows, int& z, bool& text) {
  const int bh = s / (p.T + 1);
  const int t = s % (p.T + 1);
  text = (t == 0);
  rows = text ? p.n_txt : p.n;
  z = text ? bh : bh * p.T + (t - 1);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Row i, K-chunk c (4 tf32 values) of a K-major, non-swizzled operand: 8-row
// core matrices of 128 bytes (SBO = 128), the two K-chunks 2 KB apart (LBO).
__device__ __forceinline__ void store_op(uint8_t* op, int i, const float (&v)[8]) {
  *reinterpret_cast<float4*>(op + i * 16) = make_float4(v[0], v[1], v[2], v[3]);
  *reinterpret_cast<float4*>(op + 2048 + i * 16) = make_float4(v[4], v[5], v[6], v[7]);
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1) gramfactor_tc_kernel(const __grid_constant__ GramFactorParams p) {
  using Cfg = GramCfg<kF8>;
  constexpr int kChunk = Cfg::kChunk;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = base;
  uint8_t* ostage = base + kStages * kStageBytes;   // 2 x B staging chunk
  uint8_t* ops0 = ostage + 2 * kOutChunk;           // per factor group: Y hi | Y lo
  float* psm0 = reinterpret_cast<float*>(ops0 + kFacGroups * 2 * kOp);   // per group: the pivot block
  Shared& sh = *reinterpret_cast<Shared*>(psm0 + kFacGroups * 64);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int slots = p.BH * (p.T + 1);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    mbar_init(&sh.gdone, 1);
    mbar_init(&sh.bfree, 128);
    for (int i = 0; i < kARegions; ++i) mbar_init(&sh.tempty[i], 128);
    for (int g = 0; g < kFacGroups; ++g) {
      mbar_init(&sh.aready[g], 128);
      mbar_init(&sh.fin[g], 128);
      mbar_init(&sh.upd[g], 1);
      mbar_init(&sh.fdone[g], 1);
    }
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.never, 1);
    sh.bad = 0;
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
    tma_prefetch_desc(&p.mB);
    if (p.n_txt > 0) {
      tma_prefetch_desc(&p.mKt);
      tma_prefetch_desc(&p.mVt);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  griddep_launch_dependents();   // the scan's CTAs may take SMs as this grid's finish

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
        const TokPos q = tok_pos(p.g, z, text);
        const CUtensorMap* mk = text ? &p.mKt : &p.mK;
        const CUtensorMap* mv = text ? &p.mVt : &p.mV;
        for (int r0 = 0; r0 < rows; r0 += kChunk) {
          if (!mbar_wait(&sh.empty[stage], phase ^ 1)) {
            set_abort(sh, p.err);
            break;
          }
          uint8_t* st = stages + stage * kStageBytes;
          mbar_expect_tx(&sh.full[stage], kStageBytes);
#pragma unroll
          for (int b = 0; b < Cfg::kBoxes; ++b) {   // features 64 b.. (bf16), or all 128 (e4m3)
            tok_load(st + b * Cfg::kBox, mk, &sh.full[stage], p.g, q, 64 * b, r0, pol);
            tok_load(st + kHalfStage + b * Cfg::kBox, mv, &sh.full[stage], p.g, q, 64 * b, r0, pol);
          }
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (aborted(sh)) {
        // Error path: the chunks that may still be in flight land first.
        for (int c = issued > kStages ? issued - kStages : 0; c < issued; ++c)
          mbar_wait(&sh.full[c % kStages], (c / kStages) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ Gram MMAs
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t sbase = smem_u32(stages);
      int j = 0;
      for (int s = blockIdx.x; s < slots && !aborted(sh); s += gridDim.x, ++j) {
        int rows, z;
        bool text;
        slot_info(p, s, rows, z, text);
        const int reg = j % kARegions;
        // The A region's previous slot has had its M written; the B region is drained.
        if (!mbar_wait(&sh.tempty[reg], ((j / kARegions) & 1) ^ 1) || !mbar_wait(&sh.bfree, (j & 1) ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        tc_fence_after();
        const uint32_t da = tmem + reg * 128, db = tmem + kBCol;
        bool first = true;
        for (int r0 = 0; r0 < rows; r0 += kChunk) {
          const bool stall = p.stall == VDA_TEST_STALL_GRAM_STAGE && blockIdx.x == 0 && j == 0 && r0 == 0;
          if (!mbar_wait_or_stall(&sh.full[stage], phase, &sh.never, stall)) {
            set_abort(sh, p.err);
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * kStageBytes;
#pragma unroll
          for (int k = 0; k < kChunk / Cfg::kKTok; ++k) {
            // kKTok tokens = kKTok rows of 128 bytes, MN-major (features
            // contiguous).  bf16: MN blocks of 64 features one box apart;
            // e4m3: one 128-feature block.  K's rows first, then V's.
            const uint64_t dk = smem_desc(sa + k * Cfg::kKTok * 128, Cfg::kBox, 1024, kSwizzle128B);
            const uint64_t dv = smem_desc(sa + kHalfStage + k * Cfg::kKTok * 128, Cfg::kBox, 1024, kSwizzle128B);
            if constexpr (kF8) {
              mma_f8_ss(da, dk, dk, kIdescGram8, first ? 0u : 1u);   // A = K^T K
              mma_f8_ss(db, dk, dv, kIdescGram8, first ? 0u : 1u);   // B = K^T V
            } else {
              mma_bf16_ss(da, dk, dk, kIdescGram, first ? 0u : 1u);
              mma_bf16_ss(db, dk, dv, kIdescGram, first ? 0u : 1u);
            }
            first = false;
          }
          mma_commit(&sh.empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (aborted(sh)) break;
        mma_commit(&sh.gdone);   // with no tokens this only marks the slot (A = lambda I, B = 0)
      }
      // Make sure no MMA is still running before TMEM is released.
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ service warps
    // Per slot, in order: B_t out (TMEM -> swizzled 32-column chunks -> TMA
    // stores), lambda onto A's diagonal in TMEM, hand A to the slot's factor
    // group; then, once the previous slot's sweep is complete, M of that slot
    // out of TMEM into global memory, and its A region back to the Gram.
    const int quarter = warp % 4;            // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;     // feature index i of D
    const bool leader = (warp == 2 && lane == 0);
    int nst = 0;
    auto write_m = [&](int s, int reg) {    // M = lambda (2I - A_final), row `row`, bf16 hi/lo
      const uint32_t trow = tmem + reg * 128 + ((uint32_t)(quarter * 32) << 16);
      uint8_t* hi = p.M + (size_t)s * 65536;
      uint8_t* lo = hi + 32768;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(trow + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {         // 8 columns per 16-byte chunk
          float h[8], l8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int col = c * 32 + q * 8 + e;
            const float m = p.lam * ((col == row ? 2.f : 0.f) - __uint_as_float(r[q * 8 + e]));
            h[e] = __bfloat162float(__float2bfloat16_rn(m));
            l8[e] = m - h[e];
          }
          const int chunk = c * 4 + q;         // 0..15
          const uint32_t off = (chunk / 8) * 16384u + sw128(row, chunk % 8);
          *reinterpret_cast<uint4*>(hi + off) = make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]),
                                                           pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7]));
          *reinterpret_cast<uint4*>(lo + off) = make_uint4(pack_bf16(l8[0], l8[1]), pack_bf16(l8[2], l8[3]),
                                                           pack_bf16(l8[4], l8[5]), pack_bf16(l8[6], l8[7]));
        }
      }
    };
    // M of slot number jm (this CTA's order) once its group's sweep is complete.
    auto finish_m = [&](int jm, int sm) -> bool {
      const int g = jm % kFacGroups;
      const bool ok = !aborted(sh) && mbar_wait(&sh.fin[g], (jm / kFacGroups) & 1);
      if (!ok && !aborted(sh)) set_abort(sh, p.err);
      if (named_bar_or(kEpiBar, 128, !ok)) return false;   // one decision for the four warps
      tc_fence_after();
      write_m(sm, jm % kARegions);
      tc_fence_before();
      mbar_arrive(&sh.tempty[jm % kARegions]);
      return true;
    };
    int prev_s = -1;
    int j = 0;
    bool live = true;
    for (int s = blockIdx.x; s < slots; s += gridDim.x, ++j) {
      const int reg = j % kARegions;
      int rows, z;
      bool text;
      slot_info(p, s, rows, z, text);
      const bool stall = p.stall == VDA_TEST_STALL_SERVICE_GRAM && blockIdx.x == 0 && j == 0;
      bool ok = !aborted(sh) && mbar_wait_or_stall(&sh.gdone, j & 1, &sh.never, stall);
      if (!ok && !aborted(sh)) set_abort(sh, p.err);
      if (named_bar_or(kEpiBar, 128, !ok)) {
        live = false;
        break;
      }
      tc_fence_after();
      const uint32_t tq = tmem + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
      for (int chunk = 0; chunk < 4; ++chunk) {
        uint32_t r[32];
        if (rows > 0) {
          tmem_ld_32x32b_x32(tq + kBCol + chunk * 32, r);
          tmem_ld_wait();
        } else {  // no tokens: B = 0
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = 0u;
        }
        uint8_t* stg = ostage + (nst & 1) * kOutChunk;
        if (leader) bulk_wait_read<1>();      // the store two chunks back has read this buffer
        named_bar_sync(kEpiBar, 128);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          *reinterpret_cast<uint4*>(stg + sw128(row, q)) =
              make_uint4(__float_as_uint(p.b_scale * __uint_as_float(r[4 * q])),
                         __float_as_uint(p.b_scale * __uint_as_float(r[4 * q + 1])),
                         __float_as_uint(p.b_scale * __uint_as_float(r[4 * q + 2])),
                         __float_as_uint(p.b_scale * __uint_as_float(r[4 * q + 3])));
        fence_proxy_async_smem();
        named_bar_sync(kEpiBar, 128);
        if (leader) {
          tma_store_2d(&p.mB, stg, chunk * 32, s * 128);
          bulk_commit();
        }
        ++nst;
      }
      tc_fence_before();
      mbar_arrive(&sh.bfree);
      // lambda on the diagonal (A = lambda I when the slot has no tokens).
      {
        const uint32_t trow = tq + reg * 128;
        uint32_t r[32];
        const int c0 = (row / 32) * 32;
        if (rows > 0) {
          tmem_ld_32x32b_x32(trow + c0, r);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = 0u;
          uint32_t zr[32];
#pragma unroll
          for (int q = 0; q < 32; ++q) zr[q] = 0u;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (c * 32 != c0) tmem_st_32x32b_x32(trow + c * 32, zr);
        }
        if (kF8 && rows > 0) {
          // e4m3: the chain holds K8^T K8 of the stored keys; A in the values'
          // units is a_scale times that, so the sweep sees A at its true
          // scale (its diagonal trick keeps 2 - (A^{-1})_ii, which needs A^{-1}
          // of the true size to keep its digits).
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            if (c * 32 == c0) continue;
            uint32_t o[32];
            tmem_ld_32x32b_x32(trow + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int q = 0; q < 32; ++q) o[q] = __float_as_uint(p.a_scale * __uint_as_float(o[q]));
            tmem_st_32x32b_x32(trow + c * 32, o);
          }
#pragma unroll
          for (int q = 0; q < 32; ++q) r[q] = __float_as_uint(p.a_scale * __uint_as_float(r[q]));
        }
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (q == row - c0) r[q] = __float_as_uint(__uint_as_float(r[q]) + p.lam);
        tmem_st_32x32b_x32(trow + c0, r);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&sh.aready[j % kFacGroups]);
      if (prev_s >= 0 && !finish_m(j - 1, prev_s)) {
        live = false;
        break;
      }
      prev_s = s;
    }
    if (live && prev_s >= 0) finish_m(j - 1, prev_s);   // the same for the four warps
    if (leader) bulk_wait<0>();               // B stores complete before exit
  } else {
    // ------------------------------------------------------------ factor groups
    // Group g sweeps this CTA's slots g, g + kFacGroups, ...: while one group
    // waits on its update MMAs the other factors its pivot block.
    const int g = (warp - 6) / 4;
    const int i = (warp % 4) * 32 + lane;    // row of A = TMEM lane (warp % 4 = lane quarter)
    const bool issuer = ((warp - 6) % 4 == 0 && lane == 0);   // first thread of the group
    const int bar = kFacBar0 + g;
    uint8_t* ops = ops0 + g * 2 * kOp;
    float (*psm)[8] = reinterpret_cast<float (*)[8]>(psm0 + g * 64);
    const uint32_t opaddr = smem_u32(ops);
    int nslot = 0;                            // slots swept by this group
    int j = g;                                // this CTA's slot number
    for (int s = blockIdx.x + g * gridDim.x; s < slots; s += kFacGroups * gridDim.x, ++nslot, j += kFacGroups) {
      const int reg = j % kARegions;
      bool ok = !aborted(sh) && mbar_wait(&sh.aready[g], nslot & 1);
      if (!ok && !aborted(sh)) set_abort(sh, p.err);
      if (named_bar_or(bar, 128, !ok)) break;
      tc_fence_after();
      const uint32_t trow = tmem + reg * 128 + ((uint32_t)((warp % 4) * 32) << 16);

      bool bad = false;
      int steps_issued = 0;
#pragma unroll 1
      for (int K = 0; K < 16; ++K) {
        if (K > 0) {
          const bool stall =
              p.stall == VDA_TEST_STALL_FACTOR_UPDATE && blockIdx.x == 0 && g == 0 && nslot == 0 && K == 1;
          const bool okw = mbar_wait_or_stall(&sh.upd[g], (K - 1) & 1, &sh.never, stall);
          if (!okw) set_abort(sh, p.err);
          if (named_bar_or(bar, 128, !okw)) break;   // the same for every thread
          tc_fence_after();
        }
        float x[8];
        {
          uint32_t r[8];
          tmem_ld_32x32b_x8(trow + 8 * K, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 8; ++q) x[q] = __uint_as_float(r[q]);
        }
        // ---- P = L L^T.  The 8 rows of the pivot block publish their pivot
        // columns; every thread factors P itself, in registers (rsqrt, no
        // divides; the same operations in the same order in every thread).
        if ((i >> 3) == K) {
          *reinterpret_cast<float4*>(&psm[i & 7][0]) = make_float4(x[0], x[1], x[2], x[3]);
          *reinterpret_cast<float4*>(&psm[i & 7][4]) = make_float4(x[4], x[5], x[6], x[7]);
        }
        named_bar_sync(bar, 128);
        float l[8][8];     // lower triangle: P, then L
        float dinv[8];     // 1 / L_jj
#pragma unroll
        for (int r = 0; r < 8; ++r) {
#pragma unroll
          for (int c = 0; c <= r; ++c) l[r][c] = psm[r][c];
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const float piv = l[jj][jj];
          bad |= !(piv > 0.f) || !isfinite(piv);
          const float rs = rsqrtf(piv);
          dinv[jj] = rs;
#pragma unroll
          for (int r = jj + 1; r < 8; ++r) l[r][jj] *= rs;
#pragma unroll
          for (int r = jj + 1; r < 8; ++r) {
#pragma unroll
            for (int c = jj + 1; c <= r; ++c) l[r][c] = fmaf(-l[r][jj], l[c][jj], l[r][c]);
          }
        }
        // ---- X~ (row i) and Y = X~ L^{-T}: forward substitution L y = x~.
        if ((i >> 3) == K) {
#pragma unroll
          for (int q = 0; q < 8; ++q) x[q] -= (q == (i & 7)) ? 1.f : 0.f;   // static indices only
        }
        float y[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float acc = x[q];
#pragma unroll
          for (int m = 0; m < q; ++m) acc = fmaf(-l[q][m], y[m], acc);
          y[q] = acc * dinv[q];
        }
        // ---- tf32 hi + lo operand (row i)
        {
          float yh[8], yl[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            yh[q] = to_tf32(y[q]);
            yl[q] = to_tf32(y[q] - yh[q]);
          }
          store_op(ops + 0 * kOp, i, yh);
          store_op(ops + 1 * kOp, i, yl);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        named_bar_sync(bar, 128);
        if (issuer) {
          tc_fence_after();
          // A -= Y Y^T: Y is the A operand (M x K) and, read K-major from the
          // same rows, the B operand (K x N).  Three tf32 passes: hi hi, hi lo,
          // lo hi; the lo lo product is below float32 rounding of the update.
          const uint64_t yhi = smem_desc(opaddr + 0 * kOp, 2048, 128, kSwizzleNone);
          const uint64_t ylo = smem_desc(opaddr + 1 * kOp, 2048, 128, kSwizzleNone);
          const uint32_t d = tmem + reg * 128;
          mma_tf32_ss(d, yhi, yhi, kIdescUpd, 1u);
          mma_tf32_ss(d, yhi, ylo, kIdescUpd, 1u);
          mma_tf32_ss(d, ylo, yhi, kIdescUpd, 1u);
          mma_commit(&sh.upd[g]);
        }
        ++steps_issued;
      }
      if (bad && i == 0) sh.bad = 1;   // every thread saw the same pivots
      // One more commit covers every update MMA issued for this slot; wait for
      // it (bounded), also on the error path, before the buffer is handed on.
      if (issuer) mma_commit(&sh.fdone[g]);
      ok = mbar_wait(&sh.fdone[g], nslot & 1) && steps_issued == 16;
      if (!ok && !aborted(sh)) set_abort(sh, p.err);
      if (named_bar_or(bar, 128, !ok)) break;
      tc_fence_before();
      mbar_arrive(&sh.fin[g]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0 && sh.bad) atomicOr(p.err, kDevErrNotSpd);
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gramfactor_tc(const vda_problem& p, const void* K, const void* V, const void* Kt, const void* Vt,
                                 float* M, float* Bm, unsigned* err, cudaStream_t st) {
  if (p.d_k != 128 || p.d_v != 128) return cudaErrorInvalidValue;
  const bool f8 = p.dtype == VDA_DTYPE_E4M3;
  const int esz = f8 ? 1 : 2;
  const int chunk = f8 ? GramCfg<true>::kChunk : GramCfg<false>::kChunk;
  GramFactorParams prm;
  memset(&prm, 0, sizeof(prm));
  const int BH = p.B * p.H;
  if (!make_tok_map(&prm.mK, K, p.layout, p.B, p.H, p.T, p.n, chunk, esz) ||
      !make_tok_map(&prm.mV, V, p.layout, p.B, p.H, p.T, p.n, chunk, esz))
    return cudaErrorInvalidValue;
  if (p.n_txt > 0 && (!make_tok_map(&prm.mKt, Kt, p.layout, p.B, p.H, 1, p.n_txt, chunk, esz) ||
                      !make_tok_map(&prm.mVt, Vt, p.layout, p.B, p.H, 1, p.n_txt, chunk, esz)))
    return cudaErrorInvalidValue;
  prm.g = TokGeom{p.layout, p.H, p.T};
  const long long rows = (long long)BH * (p.T + 1) * 128;
  if (!make_f32_rows_map(&prm.mB, Bm, rows, 128)) return cudaErrorInvalidValue;
  prm.M = reinterpret_cast<uint8_t*>(M);
  prm.err = err;
  prm.BH = BH;
  prm.T = p.T;
  prm.n = p.n;
  prm.n_txt = p.n_txt;
  // e4m3 inputs hold K / scale_k and V / scale_v: the chains accumulate the
  // stored values' products, and the service warps scale them to the values'
  // units (A by scale_k^2, B by scale_k scale_v) before anything else reads them.
  prm.lam = p.lambda;
  prm.a_scale = f8 ? p.scale_k * p.scale_k : 1.f;
  prm.b_scale = f8 ? p.scale_k * p.scale_v : 1.f;
  prm.stall = p.test_stall;
  const size_t smem = 1024 + kStages * kStageBytes + 2 * kOutChunk + kFacGroups * (2 * kOp + 8 * 8 * 4) + sizeof(Shared);
  auto kern = f8 ? gramfactor_tc_kernel<true> : gramfactor_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int slots = BH * (p.T + 1);
  const int grid = slots < sms ? slots : sms;
  kern<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
