// Gated readout on tcgen05 tensor cores:
//     O_t = sigmoid(G_t) * (Q_t (S^f_t + S^b_t))
// ("VDN-MiniMax-H3" (aiezz.com), section 03, gate fusion item: a
// content-dependent sigmoid gate on the branch output).  bfloat16 Q, G, O and
// states, d = 128; or e4m3 Q and G with per-tensor scales (O and states
// bfloat16): each Q tile is widened exactly to bfloat16 into tensor memory,
// where the MMA reads its A operand (an MMA takes one element type for both
// operands, and the states stay bfloat16), and G is widened in the epilogue.
//
// Precision: Q is exact in bf16; the scan hands over S^f and S^b as bf16,
// and O = sigmoid(G) * (Q S^f + Q S^b) takes two MMA passes accumulated in
// float32 (about 2e-3 relative error in O with its bf16 rounding, against
// 1.7e-3 for that rounding alone).
//
// Design (persistent, one CTA per SM, 18 warps), work = 128-row tiles of every
// frame, a contiguous range of tiles per CTA:
//   warp 0      TMA producer: Q tiles and G tiles (2-stage rings), each tile
//               as two 64-feature boxes with the 128-byte swizzle.
//   warp 1      TMEM (2 x 128 columns) and the MMAs (one thread).
//   warps 2..9  per tile: TMEM -> registers, gate from the G tile (sigmoid
//               as (1 + tanh(g/2)) / 2, one special-function op), O written
//               over the G tile in shared memory, then a TMA store per
//               64-column half.  Warps 2..5 take columns 0..63 and warps 6..9
//               columns 64..127 (two warps per TMEM lane quarter).
//   warps 10..17 S^f and S^b of the next frame, streamed by bulk copies
//               through a 2-slot shared-memory ring into registers a frame
//               ahead, then written into the MMA's B operand buffer as soon
//               as the MMAs release it.
//   e4m3 inputs: Q and G tiles are half the size, so their rings are 3 and
//               4 deep (about the bytes in flight of bf16).  The epilogue warps
//               form two groups that take alternate tiles over all 128
//               columns (the tile's parity picks its accumulator and its
//               64-column A slot); each group also widens its next tile's Q,
//               each thread its own row, straight into its A slot, and sends
//               O out through its two 8 KB staging boxes in turn (32-column
//               TMA stores).
// Every wait is bounded (see sm100.cuh); a wait that runs out sets the timeout
// bit of the error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kQStages = 2;                  // bf16 input rings (32 KB tiles)
constexpr int kGStages = 2;
constexpr int kQStages8 = 3;                 // e4m3 input rings (16 KB tiles)
constexpr int kGStages8 = 4;
constexpr int kRows = 128;                   // tokens per tile
constexpr int kBox = kRows * 64 * 2;         // 128 rows x 64 features bf16: 16 KB
constexpr int kTile = 2 * kBox;              // 32 KB
constexpr int kSig = 2 * kTile;              // S^f and S^b (bf16 operands), 32 KB each
constexpr int kPieceRows = 16;               // S^f, S^b streamed in 16-row pieces
constexpr int kPieces = 128 / kPieceRows;    // 8 pieces per frame
constexpr int kPieceHalf = kPieceRows * 128 * 2;   // 4 KB of S^f (or S^b) per piece
constexpr int kPiece = 2 * kPieceHalf;       // one staging slot: S^f piece | S^b piece
constexpr int kThreads = 576;              // 2 control warps + 8 epilogue warps + 8 prep warps
// e4m3 inputs: Q and G tiles are 16 KB (one 128-byte row per token).
constexpr int kTile8 = kRows * 128;          // 16 KB
constexpr int kOStage = kRows * 32 * 2;      // 128 rows x 32 bf16 columns: 8 KB
constexpr uint32_t kTmemCols = 256;          // two 128-column accumulators
constexpr uint32_t kTmemCols8 = 512;         // e4m3: and two 64-column A slots (the widened Q)
constexpr uint32_t kACol = 256;
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ true);

struct ReadoutTcParams {
  CUtensorMap mQ, mG, mO;
  CUtensorMap mSF, mSB;      // the same states as tiles: 64 columns x 128 rows, 128-byte swizzle
  const __nv_bfloat16* SF;   // [frames][128][128]
  const __nv_bfloat16* SB;
  unsigned* err;
  int units;       // B*H*T frames
  int n;           // tokens per frame
  int tiles_per_unit;
  TokGeom g;       // the layout of Q, G and O
  int stall;       // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
  float q_scale;   // e4m3 inputs: the values Q and G stand for are q_scale Q and g_scale G (1 for bf16)
  float g_scale;
};

struct Shared {
  uint64_t q_full[kQStages8], q_empty[kQStages8];
  uint64_t g_full[kGStages8], g_empty[kGStages8];
  uint64_t t_full[2], t_empty[2];
  uint64_t a_full[2];   // e4m3: the widened Q tiles in tensor memory (the MMA's A operand)
  uint64_t sig_full, sig_empty;
  uint64_t p_full[2];   // S staging slots
  uint64_t s0_full;     // the first frame's states, loaded straight into the operand buffer
  uint64_t drain;
  uint64_t never;       // testing hook: nothing arrives on it
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

// Byte offset of 16-byte chunk `chunk` (0..3) of row `row` in a 64-byte-
// swizzled box (rows of 64 bytes, 512-byte atoms, 512-byte aligned).
__device__ __forceinline__ uint32_t sw64(uint32_t row, uint32_t chunk) {
  return row * 64u + ((chunk ^ ((row >> 1) & 3u)) << 4);
}

// Two e4m3 values (low byte first) to two f16 (exact: every e4m3 value is a
// normal f16 or zero).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint16_t x) {
  uint32_t r;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(x));
  return r;
}
// Two f16 that came from e4m3 (normal or zero) to two bf16, exactly: the f16
// exponent and top mantissa bits moved into bf16 position read as the value
// times 2^-112 (a normal bf16), and the product with 2^112 is exact.
__device__ __forceinline__ uint32_t f16x2_to_bf16x2_exact(uint32_t h) {
  const uint32_t bits = ((h >> 3) & 0x0FFF0FFFu) | (h & 0x80008000u);
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(bits), "r"(0x77807780u));
  return r;
}

template <bool kF8>
__global__ void __launch_bounds__(kThreads, 1) readout_tc_kernel(const __grid_constant__ ReadoutTcParams p) {
  constexpr int kQT = kF8 ? kTile8 : kTile;         // bytes of one Q (or G) input tile
  constexpr int kQS = kF8 ? kQStages8 : kQStages;   // ring depths
  constexpr int kGS = kF8 ? kGStages8 : kGStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sig = base;                              // S^f | S^b
  uint8_t* qbuf = base + kSig;                      // kQS input tiles
  uint8_t* gbuf = qbuf + kQS * kQT;                 // kGS tiles (bf16: G in, O out; e4m3: G in)
  uint8_t* sstage = gbuf + kGS * kQT;               // 2 S staging slots
  uint8_t* ostage = sstage + 2 * kPiece;            // e4m3: two 8 KB O staging boxes per column half
  Shared& sh = *reinterpret_cast<Shared*>(ostage + (kF8 ? 4 * kOStage : 0));

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long total = (long long)p.units * p.tiles_per_unit;
  const int t_begin = (int)(total * blockIdx.x / gridDim.x);
  const int t_end = (int)(total * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQS; ++i) {
      mbar_init(&sh.q_full[i], 1);
      mbar_init(&sh.q_empty[i], kF8 ? 128 : 1);   // bf16: the tile's MMAs; e4m3: the widening group
    }
    for (int i = 0; i < 2; ++i) mbar_init(&sh.a_full[i], 128);
    for (int i = 0; i < kGS; ++i) {
      mbar_init(&sh.g_full[i], 1);
      mbar_init(&sh.g_empty[i], kF8 ? 128 : 2);   // bf16: one arrival per stored half; e4m3: per reader
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.t_full[i], 1);
      mbar_init(&sh.t_empty[i], kF8 ? 128 : 256);   // e4m3: the tile's group; bf16: both halves
    }
    mbar_init(&sh.sig_full, 256);   // the 8 prep warps
    mbar_init(&sh.sig_empty, 1);
    mbar_init(&sh.p_full[0], 1);
    mbar_init(&sh.p_full[1], 1);
    mbar_init(&sh.s0_full, 1);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.never, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kF8 ? kTmemCols8 : kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&p.mQ);
    tma_prefetch_desc(&p.mG);
    tma_prefetch_desc(&p.mO);
    tma_prefetch_desc(&p.mSF);
    tma_prefetch_desc(&p.mSB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int qs = 0, gs = 0;
      uint32_t qph = 0, gph = 0;
      int q_issued = 0, g_issued = 0;
      int pos_u = -1;
      TokPos q{};
      for (int tile = t_begin; tile < t_end && !aborted(sh); ++tile) {
        const int u = tile / p.tiles_per_unit;
        const int y = (tile % p.tiles_per_unit) * kRows;
        if (u != pos_u) {
          q = tok_pos(p.g, u, false);
          pos_u = u;
        }
        if (!mbar_wait(&sh.q_empty[qs], qph ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        mbar_expect_tx(&sh.q_full[qs], kQT);
        tok_load(qbuf + qs * kQT, &p.mQ, &sh.q_full[qs], p.g, q, 0, y, pol);
        if (!kF8) tok_load(qbuf + qs * kQT + kBox, &p.mQ, &sh.q_full[qs], p.g, q, 64, y, pol);
        ++q_issued;
        if (++qs == kQS) { qs = 0; qph ^= 1; }
        if (!mbar_wait(&sh.g_empty[gs], gph ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        mbar_expect_tx(&sh.g_full[gs], kQT);
        tok_load(gbuf + gs * kQT, &p.mG, &sh.g_full[gs], p.g, q, 0, y, pol);
        if (!kF8) tok_load(gbuf + gs * kQT + kBox, &p.mG, &sh.g_full[gs], p.g, q, 64, y, pol);
        ++g_issued;
        if (++gs == kGS) { gs = 0; gph ^= 1; }
      }
      if (aborted(sh)) {  // let the loads still in flight land before exit
        for (int c = q_issued > kQS ? q_issued - kQS : 0; c < q_issued; ++c)
          mbar_wait(&sh.q_full[c % kQS], (c / kQS) & 1);
        for (int c = g_issued > kGS ? g_issued - kGS : 0; c < g_issued; ++c)
          mbar_wait(&sh.g_full[c % kGS], (c / kGS) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int qs = 0, tb = 0;
      uint32_t qph = 0, tph = 0, sph = 0;
      int cur_u = -1;
      const uint32_t qaddr = smem_u32(qbuf);
      const uint32_t saddr = smem_u32(sig);
      for (int tile = t_begin; tile < t_end && !aborted(sh); ++tile) {
        const int u = tile / p.tiles_per_unit;
        if (u != cur_u) {
          if (!mbar_wait(&sh.sig_full, sph)) { set_abort(sh, p.err); break; }
          sph ^= 1;
          cur_u = u;
        }
        if (!mbar_wait(&sh.t_empty[tb], tph ^ 1)) { set_abort(sh, p.err); break; }
        // The A operand: the bf16 Q tile, or (e4m3) its widened copy in
        // tensor memory (A slot = tile parity, as the accumulator).
        const bool stall = p.stall == VDA_TEST_STALL_READOUT_TILE && blockIdx.x == 0 && tile == t_begin;
        uint64_t* afull = kF8 ? &sh.a_full[tb] : &sh.q_full[qs];
        if (!mbar_wait_or_stall(afull, kF8 ? tph : qph, &sh.never, stall)) { set_abort(sh, p.err); break; }
        tc_fence_after();
        const uint32_t d = tmem + tb * 128;
        const uint32_t qa = qaddr + qs * kTile;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // B: S^f or S^b, MN-major; 16 rows of 128 bytes per k-step,
            // 64-column blocks 16 KB apart.
            const uint64_t b = smem_desc(saddr + pass * kTile + k * 16 * 128, kBox, 1024, kSwizzle128B);
            if constexpr (kF8) {
              // A: 16 features = 8 columns of the tile's A slot.
              mma_bf16_ts(d, tmem + kACol + tb * 64 + 8 * k, b, kIdesc, (pass | k) ? 1u : 0u);
            } else {
              // A: Q tile, K-major; 16 features = 32 bytes inside a 128-byte row.
              const uint64_t a = smem_desc(qa + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
              mma_bf16_ss(d, a, b, kIdesc, (pass | k) ? 1u : 0u);
            }
          }
        }
        // bf16: the Q tile is free.  e4m3: the widening threads free the
        // 8-bit tile, and the A slot is free once t_full has arrived.
        if (!kF8) mma_commit(&sh.q_empty[qs]);
        mma_commit(&sh.t_full[tb]);
        const bool last_of_unit = (tile + 1 == t_end) || ((tile + 1) / p.tiles_per_unit != u);
        if (last_of_unit) mma_commit(&sh.sig_empty);
        if (++qs == kQStages) { qs = 0; qph ^= 1; }
        tb ^= 1;
        if (tb == 0) tph ^= 1;
      }
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;          // 0..255
    const int quarter = warp % 4;             // TMEM lanes this warp may access
    const int row = quarter * 32 + lane;      // tile row this thread owns in TMEM
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const float hq = 0.5f * p.q_scale, hg = 0.5f * p.g_scale;
    if constexpr (kF8) {
      // e4m3: two groups of four warps take alternate tiles (the tile's
      // parity: its accumulator and its A slot), all 128 columns each, so one
      // group's gate and stores overlap the other's.  Per tile k of the group:
      // the gate from TMEM and G, O through the group's two 8 KB staging
      // boxes in turn (32 columns, 64-byte rows, TMA stores, rows past n
      // clipped), and, before its last columns are read, the group's next
      // tile's Q widened into its A slot (free: this tile's MMAs, which read
      // it, are complete), so those MMAs overlap the rest of this tile.
      const int grp = (warp - 2) / 4;
      const bool leader = et % 128 == 0;
      const uint32_t acc = tmem + grp * 128 + lane_off;
      const uint32_t aslot = tmem + kACol + grp * 64 + lane_off;
      const int K = t_end - t_begin;
      auto widen = [&](int k) -> bool {       // tile t_begin + k's Q, this thread's row
        const int qs = k % kQS;
        bool ok = !aborted(sh) && mbar_wait(&sh.q_full[qs], (k / kQS) & 1);
        if (!__all_sync(0xffffffffu, ok)) return false;   // the TMEM stores below are warp-wide
        const uint8_t* src = qbuf + qs * kQT;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {         // features 64 h .. 64 h + 63
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {       // features 64 h + 16 c .. + 15
            const uint4 v = *reinterpret_cast<const uint4*>(src + sw128(row, 4 * h + c));
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o[8 * c + 2 * e] = f16x2_to_bf16x2_exact(e4m3x2_to_f16x2((uint16_t)(wv[e] & 0xFFFFu)));
              o[8 * c + 2 * e + 1] = f16x2_to_bf16x2_exact(e4m3x2_to_f16x2((uint16_t)(wv[e] >> 16)));
            }
          }
          tmem_st_32x32b_x32(aslot + 32 * h, o);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh.q_empty[qs]);
        mbar_arrive(&sh.a_full[grp]);
        return true;
      };
      bool ok = true;
      if (grp < K) ok = widen(grp);
      for (int k = grp; k < K; k += 2) {
        const int tile = t_begin + k;
        const int u = tile / p.tiles_per_unit;
        const int y = (tile % p.tiles_per_unit) * kRows;
        const int gs = k % kGS;
        const bool stall = p.stall == VDA_TEST_STALL_READOUT_GATE && blockIdx.x == 0 && tile == t_begin + 1;
        ok = ok && !aborted(sh) && mbar_wait(&sh.t_full[grp], (k >> 1) & 1);
        ok = ok && mbar_wait_or_stall(&sh.g_full[gs], (k / kGS) & 1, &sh.never, stall);
        if (!ok) set_abort(sh, p.err);
        // One decision for the group's four warps, which meet at its named
        // barrier below: a warp that left alone would strand the others.
        if (named_bar_or(1 + grp, 128, !ok)) break;
        tc_fence_after();
        const uint8_t* g8row = gbuf + gs * kQT;
        const TokPos opos = tok_pos(p.g, u, false);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {         // 32 columns at a time
          // Before the last columns: the group's next tile into its A slot,
          // then, with the accumulator read, that tile's MMAs may start.
          if (c == 3 && k + 2 < K) ok = widen(k + 2);
          uint32_t r[32];
          tmem_ld_32x32b_x32(acc + 32 * c, r);
          tmem_ld_wait();
          if (c == 3) {
            tc_fence_before();
            mbar_arrive(&sh.t_empty[grp]);
          }
          uint4 ch[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int f0 = c * 32 + q * 8;    // features f0 .. f0 + 7: half a 16-byte chunk
            const uint2 gv = *reinterpret_cast<const uint2*>(g8row + sw128(row, f0 >> 4) + (f0 & 15));
            const uint32_t gw[2] = {gv.x, gv.y};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t h2 = e4m3x2_to_f16x2((uint16_t)(gw[e >> 1] >> (16 * (e & 1))));
              const float2 gf = __half22float2(*reinterpret_cast<const __half2*>(&h2));
              // sigmoid(g) d = (1 + tanh(g / 2)) d / 2: one special-function op.
              const float h0 = hq * __uint_as_float(r[q * 8 + 2 * e]);
              const float h1 = hq * __uint_as_float(r[q * 8 + 2 * e + 1]);
              ow[e] = pack_bf16(fmaf(h0, tanh_approx(hg * gf.x), h0), fmaf(h1, tanh_approx(hg * gf.y), h1));
            }
            ch[q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
          if (c == 3) mbar_arrive(&sh.g_empty[gs]);
          uint8_t* ostg = ostage + (2 * grp + (c & 1)) * kOStage;
          if (leader) bulk_wait_read<1>();     // the store two boxes back has read this one
          named_bar_sync(1 + grp, 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(ostg + sw64(row, q)) = ch[q];
          fence_proxy_async_smem();
          named_bar_sync(1 + grp, 128);
          if (leader) {
            tok_store(&p.mO, ostg, p.g, opos, 32 * c, y);
            bulk_commit();
          }
        }
      }
      if (leader) bulk_wait<0>();             // O stores complete before exit
    } else {
      // bf16: warps 2..5 take columns 0..63 and warps 6..9 columns 64..127
      // of every tile (two warps per TMEM lane quarter).
      const int half = (warp - 2) / 4;
      int gs = 0, tb = 0;
      uint32_t gph = 0, tph = 0;
      for (int tile = t_begin; tile < t_end; ++tile) {
        const int u = tile / p.tiles_per_unit;
        const int y = (tile % p.tiles_per_unit) * kRows;
        const bool stall = p.stall == VDA_TEST_STALL_READOUT_GATE && blockIdx.x == 0 && tile == t_begin + 1;
        bool ok = !aborted(sh) && mbar_wait(&sh.t_full[tb], tph);
        ok = ok && mbar_wait_or_stall(&sh.g_full[gs], gph, &sh.never, stall);
        if (!ok) set_abort(sh, p.err);
        // One decision for the half's four warps, which meet at its named
        // barrier below: a warp that left alone would strand the others.
        if (named_bar_or(1 + half, 128, !ok)) break;
        tc_fence_after();
        const uint32_t taddr = tmem + tb * 128 + half * 64 + lane_off;
        // G is read from, and O written over, the G tile, then stored by TMA.
        uint8_t* rowp = gbuf + gs * kTile + half * kBox;
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {           // 32 output columns per step
          uint32_t r[32];
          tmem_ld_32x32b_x32(taddr + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {          // 8 columns = one 16-byte chunk
            const uint32_t off = sw128(row, c * 4 + q);
            const uint4 gv = *reinterpret_cast<const uint4*>(rowp + off);
            const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(&gw[e]);
              // sigmoid(g) d = (1 + tanh(g / 2)) d / 2: one special-function op.
              const float h0 = hq * __uint_as_float(r[q * 8 + 2 * e]);
              const float h1 = hq * __uint_as_float(r[q * 8 + 2 * e + 1]);
              ow[e] = pack_bf16(fmaf(h0, tanh_approx(hg * __low2float(g2)), h0),
                                fmaf(h1, tanh_approx(hg * __high2float(g2)), h1));
            }
            *reinterpret_cast<uint4*>(rowp + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        }
        tc_fence_before();
        mbar_arrive(&sh.t_empty[tb]);
        fence_proxy_async_smem();
        named_bar_sync(1 + half, 128);
        if (et % 128 == 0) {   // first thread of each half stores that half
          tok_store(&p.mO, rowp, p.g, tok_pos(p.g, u, false), 64 * half, y);
          bulk_commit();
          bulk_wait_read<0>();
          mbar_arrive(&sh.g_empty[gs]);
        }
        if (++gs == kGS) { gs = 0; gph ^= 1; }
        tb ^= 1;
        if (tb == 0) tph ^= 1;
      }
      if (et % 128 == 0) bulk_wait<0>();       // O stores complete before exit
    }
  } else if (warp < 18) {
    // ------------------------------------------------------------ S prep
    // S^f and S^b (bfloat16) of each frame of this CTA's range, in order.
    // The first frame's go straight into the operand buffer, which is free
    // at the start: four TMA tile loads (64 columns x 128 rows, swizzled as
    // the MMA reads them), one round trip.  Every later frame's 8 pieces (16
    // rows of S^f and of S^b, 4 KB each, contiguous) arrive by bulk copy in a
    // 2-slot ring, issued by the first prep thread as slots free up, so no
    // global load goes through the load/store unit (a burst of them there
    // stalls the epilogue's shared-memory traffic).  Thread pt keeps row
    // 16 j + pt / 16, columns 8 (pt % 16) .. + 7 of every piece j in
    // registers; once the MMAs release the operand buffer it writes them
    // there (swizzled) and the next frame's pieces start.
    const int pt = threadIdx.x - 320;         // 0..255
    const int prow = pt / 16;                 // row inside a piece
    const int pchunk = pt % 16;               // 8-column chunk
    const int u_first = t_begin / p.tiles_per_unit;
    const int u_last = t_end > t_begin ? (t_end - 1) / p.tiles_per_unit : u_first - 1;
    const int n_pieces = (u_last - u_first) * kPieces;   // frames after the first
    auto issue = [&](int g) {                 // piece g of the sequence into slot g % 2
      const int u = u_first + 1 + g / kPieces, j = g % kPieces;
      const size_t off = ((size_t)u * 128 + (size_t)j * kPieceRows) * 128;
      uint8_t* dst = sstage + (g & 1) * kPiece;
      mbar_expect_tx(&sh.p_full[g & 1], kPiece);
      bulk_load(dst, p.SF + off, kPieceHalf, &sh.p_full[g & 1]);
      bulk_load(dst + kPieceHalf, p.SB + off, kPieceHalf, &sh.p_full[g & 1]);
    };
    int issued = 0;
    bool first_issued = false;
    if (pt == 0) griddep_wait();              // the states come from the previous kernel
    if (pt == 0 && u_first <= u_last) {
      const uint64_t pol = policy_evict_first();
      mbar_expect_tx(&sh.s0_full, kSig);
      tma_load_3d(sig, &p.mSF, &sh.s0_full, 0, 0, u_first, pol);
      tma_load_3d(sig + kBox, &p.mSF, &sh.s0_full, 64, 0, u_first, pol);
      tma_load_3d(sig + kTile, &p.mSB, &sh.s0_full, 0, 0, u_first, pol);
      tma_load_3d(sig + kTile + kBox, &p.mSB, &sh.s0_full, 64, 0, u_first, pol);
      first_issued = true;
      for (; issued < 2 && issued < n_pieces; ++issued) issue(issued);
    }
    uint32_t seph = 0;
    int g = 0;                                 // pieces consumed
    int landed = 0;                            // pieces whose copies are known to have landed
    bool s0_waited = false, stop = false;
    if (u_first <= u_last) {                   // the same for every prep thread
      // The first frame: hand the operand buffer to the MMAs once it has landed.
      const bool ok = mbar_wait(&sh.s0_full, 0);
      s0_waited = true;
      if (!ok) set_abort(sh, p.err);
      stop = named_bar_or(3, 256, !ok);        // one decision for all prep threads
      if (!stop) {
        mbar_arrive(&sh.sig_full);
        seph ^= 1;                             // the MMAs release the buffer once per frame
      }
    }
    for (int u = u_first + 1; u <= u_last && !stop; ++u) {
      if (pt == 0 && u + 1 <= u_last) {
        // Read about a frame from now: bring into L2 first.
        bulk_prefetch_l2(p.SF + (size_t)(u + 1) * 128 * 128, 128 * 128 * 2);
        bulk_prefetch_l2(p.SB + (size_t)(u + 1) * 128 * 128, 128 * 128 * 2);
      }
      uint4 sf[kPieces], sb[kPieces];
      bool ok = true;
#pragma unroll
      for (int j = 0; j < kPieces; ++j, ++g) {
        const bool stall = p.stall == VDA_TEST_STALL_READOUT_STATE && blockIdx.x == 0 && g == 0;
        ok = ok && mbar_wait_or_stall(&sh.p_full[g & 1], (g >> 1) & 1, &sh.never, stall);
        if (ok) landed = g + 1;
        const uint8_t* f = sstage + (g & 1) * kPiece + prow * 256 + pchunk * 16;
        sf[j] = *reinterpret_cast<const uint4*>(f);
        sb[j] = *reinterpret_cast<const uint4*>(f + kPieceHalf);
        named_bar_sync(3, 256);                // every prep thread is done with the slot
        if (pt == 0 && ok && issued < n_pieces) issue(issued++);
      }
      if (!ok) set_abort(sh, p.err);
      ok = ok && !aborted(sh) && mbar_wait(&sh.sig_empty, seph ^ 1);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(3, 256, !ok)) break;    // one decision for all prep threads
      seph ^= 1;
#pragma unroll
      for (int j = 0; j < kPieces; ++j) {
        const uint32_t off = (pchunk / 8) * kBox + sw128(j * kPieceRows + prow, pchunk % 8);
        *reinterpret_cast<uint4*>(sig + off) = sf[j];
        *reinterpret_cast<uint4*>(sig + kTile + off) = sb[j];
      }
      fence_proxy_async_smem();
      mbar_arrive(&sh.sig_full);
    }
    if (pt == 0 && first_issued && !s0_waited) mbar_wait(&sh.s0_full, 0);
    if (pt == 0) {   // let the copies still in flight land before exit
      for (int c = landed; c < issued; ++c) mbar_wait(&sh.p_full[c & 1], (c >> 1) & 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kF8 ? kTmemCols8 : kTmemCols);
}

}  // namespace

cudaError_t launch_readout_tc(const vda_problem& p, const void* Q, const void* G, const __nv_bfloat16* SF,
                              const __nv_bfloat16* SB, __nv_bfloat16* O, unsigned* err, cudaStream_t st) {
  const bool f8 = p.dtype == VDA_DTYPE_E4M3;
  const int esz = f8 ? 1 : 2;
  ReadoutTcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int units = p.B * p.H * p.T;
  if (!make_tok_map(&prm.mQ, Q, p.layout, p.B, p.H, p.T, p.n, kRows, esz) ||
      !make_tok_map(&prm.mG, G, p.layout, p.B, p.H, p.T, p.n, kRows, esz) ||
      !make_tok_map(&prm.mO, O, p.layout, p.B, p.H, p.T, p.n, kRows, 2, f8 ? 64 : 128) ||
      !make_bf16_rows_map(&prm.mSF, SF, 128, units, 128) || !make_bf16_rows_map(&prm.mSB, SB, 128, units, 128))
    return cudaErrorInvalidValue;
  prm.SF = SF;
  prm.SB = SB;
  prm.err = err;
  prm.units = units;
  prm.n = p.n;
  prm.tiles_per_unit = (p.n + kRows - 1) / kRows;
  prm.g = TokGeom{p.layout, p.H, p.T};
  prm.stall = p.test_stall;
  prm.q_scale = f8 ? p.scale_q : 1.f;
  prm.g_scale = f8 ? p.scale_g : 1.f;
  const size_t smem = 1024 + kSig + (f8 ? (kQStages8 + kGStages8) * kTile8 : (kQStages + kGStages) * kTile) +
                      2 * kPiece + (f8 ? 4 * kOStage : 0) + sizeof(Shared);
  auto kern = f8 ? readout_tc_kernel<true> : readout_tc_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)units * prm.tiles_per_unit;
  const int grid = (int)(tiles < sms ? tiles : sms);
  // Launched with programmatic stream serialization: its CTAs start as the
  // scan's CTAs finish (or on SMs the scan leaves free) and begin loading Q
  // and G; only the state loads wait for the scan (griddep_wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

}  // namespace vda
