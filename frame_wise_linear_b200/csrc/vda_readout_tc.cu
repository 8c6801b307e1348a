// Gated readout on tcgen05 tensor cores:
//     O_t = sigmoid(G_t) * (Q_t (S^f_t + S^b_t))
// ("VDN-MiniMax-H3" (aiezz.com), section 03, gate fusion item: a
// content-dependent sigmoid gate on the branch output).  bfloat16 Q, G, O and
// states, d = 128.
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
// Every wait is bounded (see sm100.cuh); a wait that runs out sets the timeout
// bit of the error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kQStages = 2;
constexpr int kGStages = 2;
constexpr int kRows = 128;                   // tokens per tile
constexpr int kBox = kRows * 64 * 2;         // 128 rows x 64 features bf16: 16 KB
constexpr int kTile = 2 * kBox;              // 32 KB
constexpr int kSig = 2 * kTile;              // S^f and S^b (bf16 operands), 32 KB each
constexpr int kPieceRows = 16;               // S^f, S^b streamed in 16-row pieces
constexpr int kPieces = 128 / kPieceRows;    // 8 pieces per frame
constexpr int kPieceHalf = kPieceRows * 128 * 2;   // 4 KB of S^f (or S^b) per piece
constexpr int kPiece = 2 * kPieceHalf;       // one staging slot: S^f piece | S^b piece
constexpr int kThreads = 576;              // 2 control warps + 8 epilogue warps + 8 prep warps
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kIdesc = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ true);

struct ReadoutTcParams {
  CUtensorMap mQ, mG, mO;
  CUtensorMap mSF, mSB;      // the same states as tiles: 64 columns x 128 rows, 128-byte swizzle
  const __nv_bfloat16* SF;   // [frames][128][128]
  const __nv_bfloat16* SB;
  unsigned* err;
  int units;       // B*H*T frames
  int tiles_per_unit;
  TokGeom g;       // the layout of Q, G and O
};

struct Shared {
  uint64_t q_full[kQStages], q_empty[kQStages];
  uint64_t g_full[kGStages], g_empty[kGStages];
  uint64_t t_full[2], t_empty[2];
  uint64_t sig_full, sig_empty;
  uint64_t p_full[2];   // S staging slots
  uint64_t s0_full;     // the first frame's states, loaded straight into the operand buffer
  uint64_t drain;
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

__global__ void __launch_bounds__(kThreads, 1) readout_tc_kernel(const __grid_constant__ ReadoutTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sig = base;                              // S^f | S^b
  uint8_t* qbuf = base + kSig;                      // kQStages tiles
  uint8_t* gbuf = qbuf + kQStages * kTile;          // kGStages tiles (G in, O out)
  uint8_t* sstage = gbuf + kGStages * kTile;        // 2 S staging slots
  Shared& sh = *reinterpret_cast<Shared*>(sstage + 2 * kPiece);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long total = (long long)p.units * p.tiles_per_unit;
  const int t_begin = (int)(total * blockIdx.x / gridDim.x);
  const int t_end = (int)(total * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&sh.q_full[i], 1);
      mbar_init(&sh.q_empty[i], 1);
    }
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&sh.g_full[i], 1);
      mbar_init(&sh.g_empty[i], 2);   // one arrival per stored half
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.t_full[i], 1);
      mbar_init(&sh.t_empty[i], 256);
    }
    mbar_init(&sh.sig_full, 256);   // the 8 prep warps
    mbar_init(&sh.sig_empty, 1);
    mbar_init(&sh.p_full[0], 1);
    mbar_init(&sh.p_full[1], 1);
    mbar_init(&sh.s0_full, 1);
    mbar_init(&sh.drain, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
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
        mbar_expect_tx(&sh.q_full[qs], kTile);
        tok_load(qbuf + qs * kTile, &p.mQ, &sh.q_full[qs], p.g, q, 0, y, pol);
        tok_load(qbuf + qs * kTile + kBox, &p.mQ, &sh.q_full[qs], p.g, q, 64, y, pol);
        ++q_issued;
        if (++qs == kQStages) { qs = 0; qph ^= 1; }
        if (!mbar_wait(&sh.g_empty[gs], gph ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        mbar_expect_tx(&sh.g_full[gs], kTile);
        tok_load(gbuf + gs * kTile, &p.mG, &sh.g_full[gs], p.g, q, 0, y, pol);
        tok_load(gbuf + gs * kTile + kBox, &p.mG, &sh.g_full[gs], p.g, q, 64, y, pol);
        ++g_issued;
        if (++gs == kGStages) { gs = 0; gph ^= 1; }
      }
      if (aborted(sh)) {  // let the loads still in flight land before exit
        for (int c = q_issued > kQStages ? q_issued - kQStages : 0; c < q_issued; ++c)
          mbar_wait(&sh.q_full[c % kQStages], (c / kQStages) & 1);
        for (int c = g_issued > kGStages ? g_issued - kGStages : 0; c < g_issued; ++c)
          mbar_wait(&sh.g_full[c % kGStages], (c / kGStages) & 1);
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
        if (!mbar_wait(&sh.q_full[qs], qph)) { set_abort(sh, p.err); break; }
        tc_fence_after();
        const uint32_t d = tmem + tb * 128;
        const uint32_t qa = qaddr + qs * kTile;
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // A: Q tile, K-major; 16 features = 32 bytes inside a 128-byte row.
            const uint64_t a = smem_desc(qa + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
            // B: S^f or S^b, MN-major; 16 rows of 128 bytes per k-step,
            // 64-column blocks 16 KB apart.
            const uint64_t b = smem_desc(saddr + pass * kTile + k * 16 * 128, kBox, 1024, kSwizzle128B);
            mma_bf16_ss(d, a, b, kIdesc, (pass | k) ? 1u : 0u);
          }
        }
        mma_commit(&sh.q_empty[qs]);
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
    const int half = (warp - 2) / 4;          // column half 0..63 or 64..127
    const int row = quarter * 32 + lane;      // tile row this thread owns in TMEM
    int gs = 0, tb = 0;
    uint32_t gph = 0, tph = 0;
    for (int tile = t_begin; tile < t_end; ++tile) {
      const int u = tile / p.tiles_per_unit;
      const int y = (tile % p.tiles_per_unit) * kRows;
      bool ok = !aborted(sh) && mbar_wait(&sh.t_full[tb], tph);
      ok = ok && mbar_wait(&sh.g_full[gs], gph);
      if (!ok) set_abort(sh, p.err);
      // One decision for the half's four warps, which meet at its named
      // barrier below: a warp that left alone would strand the others.
      if (named_bar_or(1 + half, 128, !ok)) break;
      tc_fence_after();
      uint8_t* gt = gbuf + gs * kTile;
      uint8_t* rowp = gt + half * kBox;
      const uint32_t taddr = tmem + tb * 128 + half * 64 + ((uint32_t)(quarter * 32) << 16);
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
            const float g0 = __low2float(g2), g1 = __high2float(g2);
            // sigmoid(g) d = (1 + tanh(g / 2)) d / 2: one special-function op.
            const float h0 = 0.5f * __uint_as_float(r[q * 8 + 2 * e]);
            const float h1 = 0.5f * __uint_as_float(r[q * 8 + 2 * e + 1]);
            ow[e] = pack_bf16(fmaf(h0, tanh_approx(0.5f * g0), h0), fmaf(h1, tanh_approx(0.5f * g1), h1));
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
      if (++gs == kGStages) { gs = 0; gph ^= 1; }
      tb ^= 1;
      if (tb == 0) tph ^= 1;
    }
    if (et % 128 == 0) bulk_wait<0>();         // O stores complete before exit
  } else {
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
        ok = ok && mbar_wait(&sh.p_full[g & 1], (g >> 1) & 1);
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
      for (int c = g; c < issued; ++c) mbar_wait(&sh.p_full[c & 1], (c >> 1) & 1);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_readout_tc(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* G,
                              const __nv_bfloat16* SF, const __nv_bfloat16* SB, __nv_bfloat16* O, unsigned* err,
                              cudaStream_t st) {
  ReadoutTcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int units = p.B * p.H * p.T;
  if (!make_tok_map(&prm.mQ, Q, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mG, G, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mO, O, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_bf16_rows_map(&prm.mSF, SF, 128, units, 128) || !make_bf16_rows_map(&prm.mSB, SB, 128, units, 128))
    return cudaErrorInvalidValue;
  prm.SF = SF;
  prm.SB = SB;
  prm.err = err;
  prm.units = units;
  prm.tiles_per_unit = (p.n + kRows - 1) / kRows;
  prm.g = TokGeom{p.layout, p.H, p.T};
  const size_t smem = 1024 + kSig + (kQStages + kGStages) * kTile + 2 * kPiece + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(readout_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
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
  return cudaLaunchKernelEx(&cfg, readout_tc_kernel, prm);
}

}  // namespace vda
