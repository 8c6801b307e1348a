// Backward of the gated readout on tcgen05 tensor cores, one pass over the
// tokens.  With S_t = S^f_t + S^b_t, P_t = Q_t S_t and s = sigmoid(G_t)
// ("VDN-MiniMax-H3" (aiezz.com), section 03, gate fusion item, differentiated):
//     dG_t = dO_t * P_t * s (1 - s),   dP_t = dO_t * s,
//     dQ_t = dP_t S_t^T,               E_t  = Q_t^T dP_t  (the states' gradient),
// bf16 Q, G, dO, dQ, dG and S_t, float32 E_t; d = 128.
//
// Per 128-token tile the MMAs compute P = Q S (A = Q K-major, B = S MN-major)
// into a TMEM buffer; the epilogue turns P, G and dO into dG (written over the
// G tile, stored by TMA) and dP (written over the dO tile, in the swizzled
// layout the tensor core reads); then dQ = dP S^T (A = dP K-major, B = S
// K-major: the same shared-memory image of S read the other way) goes into
// the same TMEM buffer and E += Q^T dP (A = Q MN-major, B = dP MN-major)
// accumulates over the frame's tiles in a TMEM block of its own.  dQ leaves
// from registers by direct stores (shared memory holds the S operand and two
// stages of Q, G and dO: 224 KB), after a shuffle transpose inside 8-lane
// groups so each store instruction writes four whole 128-byte row segments;
// E leaves the same way once per frame.
//
// Design (persistent, one CTA per SM, 10 warps); each CTA takes a contiguous
// range of whole frames, so E needs no cross-CTA reduction:
//   warp 0     TMA producer: S_t per frame, Q, G, dO tiles (2-stage rings).
//   warp 1     TMEM (3 x 128 columns for P / dQ, 128 for E) and the MMAs.
//   warps 2..9 epilogue: tile j's dG / dP, then tile j-1's dQ (its MMAs ran
//              meanwhile), and E at the end of each frame.  Two warps per
//              TMEM lane quarter, each on 64 of the 128 columns.
// Every wait is bounded (see sm100.cuh); a wait that runs out sets the timeout
// bit of the error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kRows = 128;                   // tokens per tile
constexpr int kBox = kRows * 64 * 2;         // 128 rows x 64 features bf16: 16 KB
constexpr int kTile = 2 * kBox;              // 32 KB
constexpr int kStages = 2;                   // Q, G and dO rings
constexpr int kTBufs = 3;                    // TMEM buffers for P_j, then dQ_j
constexpr uint32_t kECol = kTBufs * 128;     // TMEM columns of E
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 320;
constexpr uint32_t kIdescP = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ true);    // Q S
constexpr uint32_t kIdescDQ = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ false);  // dP S^T
constexpr uint32_t kIdescE = idesc_bf16_f32(128, 128, /*a MN*/ true, /*b MN*/ true);     // Q^T dP

struct ReadoutBwdParams {
  CUtensorMap mQ, mG, mdO, mdG;   // [frames][n][128] bf16, 64 x 128 boxes
  CUtensorMap mS;                 // [frames][128][128] bf16, 64 x 128 boxes
  const __nv_bfloat16* S;
  __nv_bfloat16* dQ;              // [frames][n][128]
  float* E;                       // [frames][128][128]
  unsigned* err;
  int frames;
  int n;
  int tiles_per_frame;
  TokGeom g;                      // the layout of Q, G, dO, dQ and dG
  int stall;                      // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t q_full[kStages], q_empty[kStages];
  uint64_t g_full[kStages], g_empty[kStages];
  uint64_t o_full[kStages], o_empty[kStages];
  uint64_t p_full[kTBufs], dp_full[kTBufs], dq_full[kTBufs], t_empty[kTBufs];
  uint64_t s_full, s_empty, e_empty;
  uint64_t drain;
  uint64_t never;                 // testing hook: nothing arrives on it
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

__global__ void __launch_bounds__(kThreads, 1) readout_bwd_tc_kernel(const __grid_constant__ ReadoutBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sbuf = base;                             // S_t of the current frame
  uint8_t* qbuf = sbuf + kTile;                     // kStages Q tiles
  uint8_t* gbuf = qbuf + kStages * kTile;           // kStages G tiles (dG out)
  uint8_t* obuf = gbuf + kStages * kTile;           // kStages dO tiles (dP in place)
  Shared& sh = *reinterpret_cast<Shared*>(obuf + kStages * kTile);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int tpf = p.tiles_per_frame;
  const int u_begin = (int)((long long)p.frames * blockIdx.x / gridDim.x);
  const int u_end = (int)((long long)p.frames * (blockIdx.x + 1) / gridDim.x);
  const int J = (u_end - u_begin) * tpf;           // tiles of this CTA

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.q_full[i], 1);
      mbar_init(&sh.q_empty[i], 1);
      mbar_init(&sh.g_full[i], 1);
      mbar_init(&sh.g_empty[i], 2);   // one arrival per stored half
      mbar_init(&sh.o_full[i], 1);
      mbar_init(&sh.o_empty[i], 1);
    }
    for (int i = 0; i < kTBufs; ++i) {
      mbar_init(&sh.p_full[i], 1);
      mbar_init(&sh.dp_full[i], 256);
      mbar_init(&sh.dq_full[i], 1);
      mbar_init(&sh.t_empty[i], 256);
    }
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.s_empty, 1);
    mbar_init(&sh.e_empty, 256);
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
    tma_prefetch_desc(&p.mQ);
    tma_prefetch_desc(&p.mG);
    tma_prefetch_desc(&p.mdO);
    tma_prefetch_desc(&p.mdG);
    tma_prefetch_desc(&p.mS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int q_issued = 0, g_issued = 0, o_issued = 0, s_issued = 0;
      TokPos q{};
      auto load_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int y) {
        mbar_expect_tx(bar, kTile);
        tok_load(dst, map, bar, p.g, q, 0, y, pol);
        tok_load(dst + kBox, map, bar, p.g, q, 64, y, pol);
      };
      for (int j = 0; j < J; ++j) {
        const int u = u_begin + j / tpf, y = (j % tpf) * kRows;
        if (j % tpf == 0) q = tok_pos(p.g, u, false);
        const int st = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1;
        if (!mbar_wait(&sh.q_empty[st], ph)) { set_abort(sh, p.err); break; }
        load_tile(qbuf + st * kTile, &p.mQ, &sh.q_full[st], y);
        ++q_issued;
        if (!mbar_wait(&sh.g_empty[st], ph)) { set_abort(sh, p.err); break; }
        load_tile(gbuf + st * kTile, &p.mG, &sh.g_full[st], y);
        ++g_issued;
        if (!mbar_wait(&sh.o_empty[st], ph)) { set_abort(sh, p.err); break; }
        load_tile(obuf + st * kTile, &p.mdO, &sh.o_full[st], y);
        ++o_issued;
        if (j % tpf == 0) {
          // S_t of this frame, once the previous frame's last dQ MMAs are done with the buffer.
          const int fr = j / tpf;
          if (fr > 0 && !mbar_wait(&sh.s_empty, (fr - 1) & 1)) { set_abort(sh, p.err); break; }
          mbar_expect_tx(&sh.s_full, kTile);
          tma_load_3d(sbuf, &p.mS, &sh.s_full, 0, 0, u, pol);
          tma_load_3d(sbuf + kBox, &p.mS, &sh.s_full, 64, 0, u, pol);
          ++s_issued;
          if (u + 1 < u_end) bulk_prefetch_l2(p.S + (size_t)(u + 1) * 128 * 128, 128 * 128 * 2);   // the next frame's
        }
      }
      if (aborted(sh)) {  // let the loads still in flight land before exit
        for (int c = q_issued > kStages ? q_issued - kStages : 0; c < q_issued; ++c)
          mbar_wait(&sh.q_full[c & 1], (c >> 1) & 1);
        for (int c = g_issued > kStages ? g_issued - kStages : 0; c < g_issued; ++c)
          mbar_wait(&sh.g_full[c & 1], (c >> 1) & 1);
        for (int c = o_issued > kStages ? o_issued - kStages : 0; c < o_issued; ++c)
          mbar_wait(&sh.o_full[c & 1], (c >> 1) & 1);
        if (s_issued > 0) mbar_wait(&sh.s_full, (s_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t saddr = smem_u32(sbuf);
      const uint32_t qaddr = smem_u32(qbuf);
      const uint32_t oaddr = smem_u32(obuf);
      // P_j = Q_j S into TMEM buffer j % 3.
      auto mma_p = [&](int j) -> bool {
        const int tb = j % kTBufs, st = j & 1;
        if (!mbar_wait(&sh.t_empty[tb], ((j / kTBufs) & 1) ^ 1)) return false;
        const bool stall = p.stall == VDA_TEST_STALL_RBWD_TILE && blockIdx.x == 0 && j == 0;
        if (!mbar_wait_or_stall(&sh.q_full[st], (j >> 1) & 1, &sh.never, stall)) return false;
        tc_fence_after();
        const uint32_t qa = qaddr + st * kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(qa + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(saddr + k * 16 * 128, kBox, 1024, kSwizzle128B);
          mma_bf16_ss(tmem + tb * 128, a, b, kIdescP, k ? 1u : 0u);
        }
        mma_commit(&sh.p_full[tb]);
        return true;
      };
      // dQ_i = dP_i S^T over P_i's TMEM columns; E += Q_i^T dP_i.
      auto mma_dq = [&](int i) -> bool {
        const int tb = i % kTBufs, st = i & 1;
        const bool first = (i % tpf) == 0, last = (i % tpf) == tpf - 1;
        if (!mbar_wait(&sh.dp_full[tb], (i / kTBufs) & 1)) return false;
        const int fr = i / tpf;
        if (first && fr > 0 && !mbar_wait(&sh.e_empty, (fr - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t da = oaddr + st * kTile;   // dP, written over dO
        const uint32_t qa = qaddr + st * kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(da + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(saddr + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          mma_bf16_ss(tmem + tb * 128, a, b, kIdescDQ, k ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(qa + k * 16 * 128, kBox, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(da + k * 16 * 128, kBox, 1024, kSwizzle128B);
          mma_bf16_ss(tmem + kECol, a, b, kIdescE, (first && k == 0) ? 0u : 1u);
        }
        mma_commit(&sh.q_empty[st]);
        mma_commit(&sh.o_empty[st]);
        mma_commit(&sh.dq_full[tb]);
        if (last) mma_commit(&sh.s_empty);
        return true;
      };
      bool ok = true;
      for (int j = 0; j < J && ok; ++j) {
        if (j % tpf == 0) {
          // A new frame: the previous frame's last tile uses the old S_t first.
          if (j > 0 && !(ok = mma_dq(j - 1))) break;
          if (!(ok = mbar_wait(&sh.s_full, (j / tpf) & 1))) break;
          ok = mma_p(j);
        } else {
          ok = mma_p(j) && mma_dq(j - 1);
        }
      }
      if (ok && J > 0) ok = mma_dq(J - 1);
      if (!ok) set_abort(sh, p.err);
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int et = threadIdx.x - 64;          // 0..255
    const int quarter = warp % 4;             // TMEM lanes this warp may access
    const int half = (warp - 2) / 4;          // columns 0..63 or 64..127
    const int row = quarter * 32 + lane;      // tile row (token) = TMEM lane
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    // Tile j: dG and dP from P_j, G_j and dO_j.
    auto epi_gate = [&](int j) -> bool {
      const int tb = j % kTBufs, st = j & 1;
      const int u = u_begin + j / tpf, y = (j % tpf) * kRows;
      bool ok = !aborted(sh) && mbar_wait(&sh.p_full[tb], (j / kTBufs) & 1);
      ok = ok && mbar_wait(&sh.g_full[st], (j >> 1) & 1);
      ok = ok && mbar_wait(&sh.o_full[st], (j >> 1) & 1);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(1 + half, 128, !ok)) return false;   // one decision per half
      tc_fence_after();
      uint8_t* grow = gbuf + st * kTile + half * kBox;
      uint8_t* orow = obuf + st * kTile + half * kBox;
      const uint32_t taddr = tmem + tb * 128 + half * 64 + lane_off;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {           // 32 columns per TMEM load
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {          // 8 columns = one 16-byte chunk
          const uint32_t off = sw128(row, c * 4 + q);
          const uint4 gv = *reinterpret_cast<const uint4*>(grow + off);
          const uint4 ov = *reinterpret_cast<const uint4*>(orow + off);
          const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
          const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
          uint32_t dgw[4], dpw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(&gw[e]);
            const __nv_bfloat162 o2 = *reinterpret_cast<const __nv_bfloat162*>(&ow[e]);
            // s = (1 + tanh(g / 2)) / 2 and s (1 - s) = (1 - tanh^2) / 4: one special-function op.
            const float t0 = tanh_approx(0.5f * __low2float(g2)), t1 = tanh_approx(0.5f * __high2float(g2));
            const float d0 = __low2float(o2), d1 = __high2float(o2);
            const float p0 = __uint_as_float(r[q * 8 + 2 * e]), p1 = __uint_as_float(r[q * 8 + 2 * e + 1]);
            dpw[e] = pack_bf16(fmaf(0.5f * d0, t0, 0.5f * d0), fmaf(0.5f * d1, t1, 0.5f * d1));
            dgw[e] = pack_bf16(0.25f * d0 * p0 * fmaf(-t0, t0, 1.f), 0.25f * d1 * p1 * fmaf(-t1, t1, 1.f));
          }
          *reinterpret_cast<uint4*>(grow + off) = make_uint4(dgw[0], dgw[1], dgw[2], dgw[3]);
          *reinterpret_cast<uint4*>(orow + off) = make_uint4(dpw[0], dpw[1], dpw[2], dpw[3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();               // dP and dG visible to the tensor core and the TMA
      mbar_arrive(&sh.dp_full[tb]);
      named_bar_sync(1 + half, 128);
      if (et % 128 == 0) {   // first thread of each half stores that half of dG
        tok_store(&p.mdG, grow, p.g, tok_pos(p.g, u, false), 64 * half, y);
        bulk_commit();
        bulk_wait_read<0>();
        mbar_arrive(&sh.g_empty[st]);
      }
      return true;
    };
    // Tile i: dQ from TMEM, stored row by row (rows past n skipped).  The
    // frame's first row and the row stride in dQ, decoded once per frame.
    int dq_u = -1;
    size_t dq_base = 0;
    const size_t rstride = tok_row_stride(p.g);
    auto epi_dq = [&](int i) -> bool {
      const int tb = i % kTBufs;
      const int u = u_begin + i / tpf, y = (i % tpf) * kRows;
      if (u != dq_u) {
        dq_base = tok_base(p.g, tok_pos(p.g, u, false), p.n, false);
        dq_u = u;
      }
      const bool stall = p.stall == VDA_TEST_STALL_RBWD_DQ && blockIdx.x == 0 && i == 0;
      bool ok = !aborted(sh) && mbar_wait_or_stall(&sh.dq_full[tb], (i / kTBufs) & 1, &sh.never, stall);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(1 + half, 128, !ok)) return false;
      tc_fence_after();
      const uint32_t taddr = tmem + tb * 128 + half * 64 + lane_off;
      // Row `row`'s 64 columns as 8 chunks, transposed across 8-lane groups:
      // chunk k of lane (g, j) is then chunk j of row 8 g + k of the quarter.
      uint4 ch[8];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          ch[c * 4 + q] = make_uint4(pack_bf16(__uint_as_float(r[8 * q]), __uint_as_float(r[8 * q + 1])),
                                     pack_bf16(__uint_as_float(r[8 * q + 2]), __uint_as_float(r[8 * q + 3])),
                                     pack_bf16(__uint_as_float(r[8 * q + 4]), __uint_as_float(r[8 * q + 5])),
                                     pack_bf16(__uint_as_float(r[8 * q + 6]), __uint_as_float(r[8 * q + 7])));
      }
      transpose8(ch, lane & 7);
      const int r0 = quarter * 32 + 8 * (lane >> 3);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int tr = y + r0 + k;             // token row; rows past n skipped
        if (tr < p.n)
          *reinterpret_cast<uint4*>(p.dQ + dq_base + tr * rstride + half * 64 + (lane & 7) * 8) = ch[k];
      }
      tc_fence_before();
      mbar_arrive(&sh.t_empty[tb]);
      return true;
    };
    // E_t of frame u (complete once the frame's last dQ is): row = d_k index.
    auto drain_e = [&](int u) {
      const uint32_t taddr = tmem + kECol + half * 64 + lane_off;
      const int r0 = quarter * 32 + 8 * (lane >> 3);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(taddr + c * 32, r);
        tmem_ld_wait();
        uint4 ch[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) ch[q] = make_uint4(r[4 * q], r[4 * q + 1], r[4 * q + 2], r[4 * q + 3]);
        transpose8(ch, lane & 7);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(p.E + ((size_t)u * 128 + r0 + k) * 128 + half * 64 + c * 32 + (lane & 7) * 4) =
              ch[k];
      }
      tc_fence_before();
      mbar_arrive(&sh.e_empty);
    };
    auto finish_dq = [&](int i) -> bool {
      if (!epi_dq(i)) return false;
      if ((i % tpf) == tpf - 1) drain_e(u_begin + i / tpf);
      return true;
    };
    for (int j = 0; j < J; ++j) {
      if (!epi_gate(j)) break;
      if (j > 0 && !finish_dq(j - 1)) break;
      if (j == J - 1) finish_dq(j);
    }
    if (et % 128 == 0) bulk_wait<0>();         // dG stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_readout_bwd_tc(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* G,
                                  const __nv_bfloat16* dO, const __nv_bfloat16* S, __nv_bfloat16* dQ,
                                  __nv_bfloat16* dG, float* E, unsigned* err, cudaStream_t st) {
  ReadoutBwdParams prm;
  memset(&prm, 0, sizeof(prm));
  const int frames = p.B * p.H * p.T;
  if (!make_tok_map(&prm.mQ, Q, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mG, G, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mdO, dO, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mdG, dG, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_bf16_rows_map(&prm.mS, S, 128, frames, 128))
    return cudaErrorInvalidValue;
  prm.S = S;
  prm.dQ = dQ;
  prm.E = E;
  prm.err = err;
  prm.frames = frames;
  prm.n = p.n;
  prm.tiles_per_frame = (p.n + kRows - 1) / kRows;
  prm.g = TokGeom{p.layout, p.H, p.T};
  prm.stall = p.test_stall;
  const size_t smem = 1024 + (1 + 3 * kStages) * kTile + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(readout_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = frames < sms ? frames : sms;
  readout_bwd_tc_kernel<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
