// The local softmax branch of the hybrid video attention on tcgen05 tensor
// cores: block-sparse scaled dot-product attention with the sliding window,
// the boundary anchors and the text, and the branch's sigmoid gate.
//
// "VDN-MiniMax-H3" (aiezz.com), section 03, local softmax branch item
// (restated in the laicaila.com page, section 技术原理): frames form blocks of
// 5, each block attends to its neighbouring blocks (a bidirectional sliding
// window), and the first and last frames are boundary anchors; the "VDN-H3"
// page (comfyui-wiki.com) adds that every frame can see them.  Text dual-
// branch injection item: in the softmax branch every frame attends to the
// whole text.  Gate fusion item: the branch has its own sigmoid gate.  Per
// (b, h) and query frame t, with S_t the tokens of frames
// {blocks t/5 - 1, t/5, t/5 + 1} u {0, T - 1} and the text:
//     O_t = sigmoid(G_t) * softmax(Q_t K_S^T / sqrt(d)) V_S
// bf16 Q, K, V, G, O; d = 128; float32 scores, softmax and accumulation.
//
// Design (persistent, one CTA per SM, 11 warps), work unit = 128 query tokens
// of one frame of one head; its key tiles are 128 tokens of one key frame (the
// last tile of a frame partial) and then of the text:
//   warps 0, 10 TMA producers: warp 0 the unit's Q tile and K tiles through a
//              3-stage ring, warp 10 V tiles through a 2-stage ring (a K tile
//              is free after its S MMAs, a V tile only after its P V).
//   warp 1     TMEM and the MMAs: S_j = Q K_j^T into one of two 128-column
//              score buffers, issued two tiles ahead, and O += P_j V_j into a
//              128-column accumulator once the softmax has written P_j, with
//              P_j read from tensor memory (two 64-column slots).
//   warps 2..9 softmax, two threads per query row (keys 0..63 and 64..127 of
//              each tile, in the same TMEM lane quarter): the row's scores
//              from TMEM, a tree for the half row's maximum, the partners'
//              maxima swapped through shared memory, the running maximum and
//              sum (log2 domain), P_j = exp2 of the scaled scores as bf16 into
//              the P slot; the accumulator is rescaled only when the maximum
//              grows by more than 2^8 (the exponentials with a stale maximum
//              stay below 2^8, and O and the sum share that maximum, so the
//              quotient is exact).  After the last tile: O / sum, times
//              sigmoid(G), each thread its half of the columns, stored from
//              registers as whole 128-byte row segments (8-lane transpose).
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kSoftmaxThreads = 256;         // 8 warps: two threads per query row
constexpr int kVWarp = 2 + kSoftmaxThreads / 32;   // the V producer, after the softmax warps
constexpr int kThreads = 32 * (kVWarp + 1);
constexpr int kKStages = 3;                  // K tiles in flight
constexpr int kVStages = 2;                  // V tiles in flight (a V tile is held until its P V is done)
constexpr int kRows = 128;                   // query and key tokens per tile
constexpr int kBox = kRows * 64 * 2;         // 128 rows x 64 features bf16: 16 KB
constexpr int kTile = 2 * kBox;              // 32 KB
constexpr int kBlock = 5;                    // frames per block of the window
constexpr float kRescale = 8.f;              // log2 growth of the maximum that forces a rescale
constexpr uint32_t kTmemCols = 512;          // S0 | S1 | O | P0 | P1
constexpr uint32_t kOCol = 256;
constexpr uint32_t kPCol = 384;              // P slots: 64 columns (128 bf16 keys) each
constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ false);   // Q K^T
constexpr uint32_t kIdescO = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ true);    // P V

struct LocalSoftmaxParams {
  CUtensorMap mQ, mK, mV;        // [B,H,T,n,128] or [B,T*n,H,128] bf16, 64 x 128 boxes
  CUtensorMap mKt, mVt;          // the text's
  const __nv_bfloat16* G;        // gate logits, the layout of Q
  __nv_bfloat16* O;
  unsigned* err;
  int BH, T, n, n_txt;
  int qtiles;                    // query tiles per frame
  float c;                       // log2(e) / sqrt(d)
  TokGeom g;
  int stall;                     // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t o_free;
  uint64_t drain;
  uint64_t never;                // testing hook: nothing arrives on it
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

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The key frames of query frame t: the window [lo, hi) of three blocks, and
// the anchors 0 and T - 1 when the window does not hold them.
struct KeyFrames {
  int lo, hi;
  bool first, last;   // anchor 0 before the window, anchor T - 1 after it
  __device__ __forceinline__ int count() const { return (hi - lo) + first + last; }
  // Frame i of the list [0 (if first)] + [lo, hi) + [T - 1 (if last)]; -1 stands for T - 1.
  __device__ __forceinline__ int frame(int i) const {
    if (first) {
      if (i == 0) return 0;
      --i;
    }
    return i < hi - lo ? lo + i : -1;
  }
};

__device__ __forceinline__ KeyFrames key_frames(int t, int T) {
  const int b = t / kBlock;
  KeyFrames k;
  k.lo = max(0, (b - 1) * kBlock);
  k.hi = min(T, (b + 2) * kBlock);
  k.first = k.lo > 0;
  k.last = k.hi < T;
  return k;
}

// Key tile j of a unit: a frame's (frame >= 0) or the text's (frame == -1),
// the tile's first token and how many of its 128 rows are keys.
struct KeyTile {
  int frame, y, valid;
  bool text;
};

__device__ __forceinline__ KeyTile key_tile(const LocalSoftmaxParams& p, const KeyFrames& kf, int j) {
  const int tpf = (p.n + kRows - 1) / kRows;
  const int nf = kf.count();
  KeyTile r;
  if (j < nf * tpf) {
    const int i = j / tpf;
    int f = kf.frame(i);
    if (f < 0) f = p.T - 1;
    r.frame = f;
    r.text = false;
    r.y = (j % tpf) * kRows;
    r.valid = min(kRows, p.n - r.y);
  } else {
    r.frame = -1;
    r.text = true;
    r.y = (j - nf * tpf) * kRows;
    r.valid = min(kRows, p.n_txt - r.y);
  }
  return r;
}

__device__ __forceinline__ int key_tiles(const LocalSoftmaxParams& p, const KeyFrames& kf) {
  return kf.count() * ((p.n + kRows - 1) / kRows) + (p.n_txt + kRows - 1) / kRows;
}

__global__ void __launch_bounds__(kThreads, 1) local_softmax_tc_kernel(const __grid_constant__ LocalSoftmaxParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qbuf = base;                      // Q tile, 32 KB
  uint8_t* kbuf = qbuf + kTile;              // kKStages K tiles
  uint8_t* vbuf = kbuf + kKStages * kTile;   // kVStages V tiles
  float* xmax = reinterpret_cast<float*>(vbuf + kVStages * kTile);   // [2 parities][2 halves][128 rows]
  float* xsum = xmax + 2 * 2 * kRows;                                 // [2 halves][128 rows]
  Shared& sh = *reinterpret_cast<Shared*>(xsum + 2 * kRows);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int units = p.BH * p.T * p.qtiles;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    for (int i = 0; i < kKStages; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], 1);
    }
    for (int i = 0; i < kVStages; ++i) {
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.s_free[i], kSoftmaxThreads);
      mbar_init(&sh.p_full[i], kSoftmaxThreads);
      mbar_init(&sh.pv_done[i], 1);
    }
    mbar_init(&sh.o_free, kSoftmaxThreads);
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

  if (warp == 0 || warp == kVWarp) {
    // ------------------------------------------------------------ producers
    // Warp 0 loads Q and the K tiles, the last warp the V tiles: a V stage is
    // freed only by its P V, late, and K loads must not queue behind it.
    if (lane == 0) {
      const bool kl = warp == 0;
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();   // a key frame serves 15 query frames
      const int stages = kl ? kKStages : kVStages;
      uint64_t* full = kl ? sh.k_full : sh.v_full;
      uint64_t* empty = kl ? sh.k_empty : sh.v_empty;
      uint8_t* ring = kl ? kbuf : vbuf;
      int issued = 0, q_issued = 0, it = 0, ui = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
        const int qt = w % p.qtiles, t = (w / p.qtiles) % p.T, bh = w / (p.qtiles * p.T);
        if (kl) {
          const TokPos qpos = tok_pos(p.g, bh * p.T + t, false);
          if (!(ok = mbar_wait(&sh.q_empty, (ui & 1) ^ 1))) break;   // the previous unit's S MMAs are done
          mbar_expect_tx(&sh.q_full, kTile);
          tok_load(qbuf, &p.mQ, &sh.q_full, p.g, qpos, 0, qt * kRows, pol_q);
          tok_load(qbuf + kBox, &p.mQ, &sh.q_full, p.g, qpos, 64, qt * kRows, pol_q);
          ++q_issued;
        }
        const KeyFrames kf = key_frames(t, p.T);
        const int J = key_tiles(p, kf);
        int cur = -2;
        TokPos kpos{};
        for (int j = 0; j < J; ++j, ++it) {
          const KeyTile kt = key_tile(p, kf, j);
          if (kt.frame != cur) {
            kpos = kt.text ? tok_pos(p.g, bh, true) : tok_pos(p.g, bh * p.T + kt.frame, false);
            cur = kt.frame;
          }
          const int st = it % stages;
          if (!(ok = mbar_wait(&empty[st], ((it / stages) & 1) ^ 1))) break;
          const CUtensorMap* map = kl ? (kt.text ? &p.mKt : &p.mK) : (kt.text ? &p.mVt : &p.mV);
          mbar_expect_tx(&full[st], kTile);
          tok_load(ring + st * kTile, map, &full[st], p.g, kpos, 0, kt.y, pol_kv);
          tok_load(ring + st * kTile + kBox, map, &full[st], p.g, kpos, 64, kt.y, pol_kv);
          ++issued;
        }
      }
      if (!ok) set_abort(sh, p.err);
      if (aborted(sh)) {   // the loads still in flight land before exit
        for (int c = issued > stages ? issued - stages : 0; c < issued; ++c) mbar_wait(&full[c % stages], (c / stages) & 1);
        if (q_issued > 0) mbar_wait(&sh.q_full, (q_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMAs
    if (lane == 0) {
      const uint32_t qa = smem_u32(qbuf), ka0 = smem_u32(kbuf), va0 = smem_u32(vbuf);
      int it = 0, ui = 0;   // global tile counter (rings, S and P buffers), unit counter
      bool ok = true;
      // S = Q K^T for the tile at position `pos` into S buffer pos & 1.
      auto issue_s = [&](int pos) -> bool {
        const int s = pos & 1, ks = pos % kKStages;
        if (!mbar_wait(&sh.s_free[s], ((pos >> 1) & 1) ^ 1)) return false;   // the softmax has read it
        if (!mbar_wait(&sh.k_full[ks], (pos / kKStages) & 1)) return false;
        tc_fence_after();
        const uint32_t ka = ka0 + ks * kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k / 4) * kBox + (k % 4) * 32;
          mma_bf16_ss(tmem + s * 128, smem_desc(qa + off, 16, 1024, kSwizzle128B),
                      smem_desc(ka + off, 16, 1024, kSwizzle128B), kIdescS, k ? 1u : 0u);
        }
        mma_commit(&sh.s_full[s]);
        mma_commit(&sh.k_empty[ks]);
        return true;
      };
      for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
        const int t = (w / p.qtiles) % p.T;
        const int J = key_tiles(p, key_frames(t, p.T));
        if (!(ok = mbar_wait(&sh.q_full, ui & 1))) break;
        // S runs two tiles ahead of P V (an MMA issue waits while the tensor
        // pipe is busy, so S_{j+2} goes in before P_j V_j, not after it).
        int ns = 0;                            // the unit's next S tile
        auto next_s = [&]() -> bool {
          if (!issue_s(it + ns)) return false;
          if (++ns == J) mma_commit(&sh.q_empty);   // the unit's last S MMAs read Q before anything after
          return true;
        };
        if (!(ok = next_s())) break;
        if (ns < J && !(ok = next_s())) break;
        for (int j = 0; j < J && ok; ++j) {
          const int pos = it + j, s = pos & 1, vs = pos % kVStages;
          // S_{j+2}: its buffer is S_j's, free once the softmax has read S_j
          if (ns < J && !(ok = next_s())) break;
          if (j == 0 && !(ok = mbar_wait(&sh.o_free, (ui & 1) ^ 1))) break;   // the previous unit's O is read
          if (!(ok = mbar_wait(&sh.p_full[s], (pos >> 1) & 1))) break;
          if (!(ok = mbar_wait(&sh.v_full[vs], (pos / kVStages) & 1))) break;
          tc_fence_after();
          // O += P V: P (K-major, 16 keys = 8 columns a step) from tensor
          // memory, V (MN-major) from shared memory.
          const uint32_t va = va0 + vs * kTile;
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_bf16_ts(tmem + kOCol, tmem + kPCol + s * 64 + 8 * k,
                        smem_desc(va + k * 16 * 128, kBox, 1024, kSwizzle128B), kIdescO, (j | k) ? 1u : 0u);
          mma_commit(&sh.pv_done[s]);
          mma_commit(&sh.v_empty[vs]);
        }
        it += J;
      }
      if (!ok) set_abort(sh, p.err);
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else if (warp < kVWarp) {
    // ------------------------------------------------------------ softmax + epilogue
    // Two threads per query row: warps 2..5 take keys (and O columns) 0..63,
    // warps 6..9 keys 64..127, in the same TMEM lane quarter.  The partners
    // swap their partial row maxima (and at the end their partial sums)
    // through shared memory at a named barrier of the quarter's two warps,
    // which is also where they decide together to stop after a timeout.
    const int quarter = warp % 4;
    const int half = (warp - 2) / 4;
    const int row = quarter * 32 + lane;       // query row = TMEM lane
    const int bar = 1 + quarter;               // named barrier of the row's two threads (64 threads)
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    const size_t rstride = tok_row_stride(p.g);
    int it = 0, ui = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
      const int qt = w % p.qtiles, t = (w / p.qtiles) % p.T, bh = w / (p.qtiles * p.T);
      const KeyFrames kf = key_frames(t, p.T);
      const int J = key_tiles(p, kf);
      const int nft = kf.count() * p.qtiles;   // the key frames' tiles (then the text's)
      int fy = 0;                              // tile of the current key frame
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < J; ++j) {
        const int pos = it + j, s = pos & 1;
        int kvalid;                            // keys in this tile
        if (j < nft) {
          kvalid = fy == p.qtiles - 1 ? p.n - fy * kRows : kRows;
          if (++fy == p.qtiles) fy = 0;
        } else {
          kvalid = min(kRows, p.n_txt - (j - nft) * kRows);
        }
        const bool stall = p.stall == VDA_TEST_STALL_SOFTMAX && blockIdx.x == 0 && pos == 0;
        ok = !aborted(sh) && mbar_wait_or_stall(&sh.s_full[s], (pos >> 1) & 1, &sh.never, stall);
        // P_j's slot is free once PV_{j-2} is done.
        ok = ok && (j < 2 || mbar_wait(&sh.pv_done[s], ((pos - 2) >> 1) & 1));
        ok = __all_sync(0xffffffffu, ok);    // the TMEM loads below are warp-wide
        float x[64];
        float mt = -INFINITY;
        if (ok) {
          tc_fence_after();
          uint32_t xr[64];
          const uint32_t sa = tmem + s * 128 + lane_off + half * 64;
          tmem_ld_32x32b_x32(sa, *reinterpret_cast<uint32_t(*)[32]>(&xr[0]));
          tmem_ld_32x32b_x32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(&xr[32]));
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&sh.s_free[s]);          // the MMAs may write the next scores here
          // raw scores; keys past the tile's valid ones excluded
#pragma unroll
          for (int e = 0; e < 64; ++e) x[e] = __uint_as_float(xr[e]);
          const int valid = kvalid - half * 64;
          if (valid < 64) {
#pragma unroll
            for (int e = 0; e < 64; ++e) x[e] = e < valid ? x[e] : -INFINITY;
          }
          // the half row's maximum by a pairwise tree (depth 6, not a chain of
          // 64), in log2 units (the scale is positive)
          float tm[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) tm[i] = fmaxf(x[2 * i], x[2 * i + 1]);
#pragma unroll
          for (int w2 = 16; w2 >= 1; w2 >>= 1) {
#pragma unroll
            for (int i = 0; i < w2; ++i) tm[i] = fmaxf(tm[2 * i], tm[2 * i + 1]);
          }
          mt = tm[0] * p.c;
        }
        if (!ok) set_abort(sh, p.err);
        xmax[(s * 2 + half) * kRows + row] = mt;
        if (named_bar_or(bar, 64, !ok)) {       // one decision for the row's two threads
          ok = false;                          // (both leave every loop: no barrier left unmet)
          break;
        }
        mt = fmaxf(mt, xmax[(s * 2 + (half ^ 1)) * kRows + row]);
        // A rescale of O needs PV_{j-1} done; the row's two threads take the
        // same decision (the same m and mt), each for its half of O.
        const bool grow = j == 0 || mt > m + kRescale;
        if (grow) {
          const float mn = fmaxf(m, mt);
          if (j >= 1) {
            ok = mbar_wait(&sh.pv_done[s ^ 1], ((pos - 1) >> 1) & 1);
            if (!ok) set_abort(sh, p.err);
            if (named_bar_or(bar, 64, !ok)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const float a = ex2(m - mn);
            l *= a;
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t r[32];
              const uint32_t oa = tmem + kOCol + lane_off + half * 64 + c * 32;
              tmem_ld_32x32b_x32(oa, r);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(a * __uint_as_float(r[e]));
              tmem_st_32x32b_x32(oa, r);
            }
            tmem_st_wait();
          }
          m = mn;
        }
        // P = 2^(c x - m) as bf16 pairs into the tile's P slot (keys 64 half ..
        // 64 half + 63 are columns 32 half .. 32 half + 31).
        {
          uint32_t pw[32];
          float lp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float v0 = ex2(fmaf(x[2 * e], p.c, -m)), v1 = ex2(fmaf(x[2 * e + 1], p.c, -m));
            lp[e & 3] += v0 + v1;
            pw[e] = pack_bf16(v0, v1);
          }
          l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
          tmem_st_32x32b_x32(tmem + kPCol + s * 64 + lane_off + half * 32, pw);
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&sh.p_full[s]);
      }
      if (!ok) break;
      // ---- epilogue: O / l times sigmoid(G), this thread's half of the
      // columns; rows past n skipped.
      const int last = it + J - 1;
      ok = !aborted(sh) && mbar_wait(&sh.pv_done[last & 1], (last >> 1) & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) set_abort(sh, p.err);
      xsum[half * kRows + row] = l;
      if (named_bar_or(bar, 64, !ok)) {
        ok = false;
        break;
      }
      const float inv = 1.f / (l + xsum[(half ^ 1) * kRows + row]);
      tc_fence_after();
      const TokPos qpos = tok_pos(p.g, bh * p.T + t, false);
      const size_t obase = tok_base(p.g, qpos, p.n, false);
      const int tok = qt * kRows + row;
      const int r0 = quarter * 32 + 8 * (lane >> 3);
      uint4 ch[8];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + kOCol + lane_off + half * 64 + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = half * 64 + c * 32 + q * 8;
          uint4 gv = make_uint4(0, 0, 0, 0);
          if (tok < p.n) gv = *reinterpret_cast<const uint4*>(p.G + obase + (size_t)tok * rstride + col);
          const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
          uint32_t ow[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 gf = __bfloat1622float2(g2[e]);
            // sigmoid(g) x = (1 + tanh(g / 2)) x / 2
            const float h0 = 0.5f * inv * __uint_as_float(r[q * 8 + 2 * e]);
            const float h1 = 0.5f * inv * __uint_as_float(r[q * 8 + 2 * e + 1]);
            ow[e] = pack_bf16(fmaf(h0, tanh_approx(0.5f * gf.x), h0), fmaf(h1, tanh_approx(0.5f * gf.y), h1));
          }
          ch[c * 4 + q] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.o_free);                 // the next unit's first PV may overwrite O
      transpose8(ch, lane & 7);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int tr = qt * kRows + r0 + k;
        if (tr < p.n) *reinterpret_cast<uint4*>(p.O + obase + (size_t)tr * rstride + half * 64 + (lane & 7) * 8) = ch[k];
      }
      it += J;
    }
    if (!ok) set_abort(sh, p.err);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_local_softmax_tc(const vda_problem& p, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                                    const __nv_bfloat16* V, const __nv_bfloat16* G, const __nv_bfloat16* Kt,
                                    const __nv_bfloat16* Vt, __nv_bfloat16* O, unsigned* err, cudaStream_t st) {
  LocalSoftmaxParams prm;
  memset(&prm, 0, sizeof(prm));
  if (!make_tok_map(&prm.mQ, Q, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mK, K, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mV, V, p.layout, p.B, p.H, p.T, p.n, kRows))
    return cudaErrorInvalidValue;
  if (p.n_txt > 0 && (!make_tok_map(&prm.mKt, Kt, p.layout, p.B, p.H, 1, p.n_txt, kRows) ||
                      !make_tok_map(&prm.mVt, Vt, p.layout, p.B, p.H, 1, p.n_txt, kRows)))
    return cudaErrorInvalidValue;
  prm.G = G;
  prm.O = O;
  prm.err = err;
  prm.BH = p.B * p.H;
  prm.T = p.T;
  prm.n = p.n;
  prm.n_txt = p.n_txt;
  prm.qtiles = (p.n + kRows - 1) / kRows;
  prm.c = 1.4426950408889634f / sqrtf((float)p.d_k);
  prm.g = TokGeom{p.layout, p.H, p.T};
  prm.stall = p.test_stall;
  const size_t smem = 1024 + (1 + kKStages + kVStages) * kTile + 3 * 2 * kRows * sizeof(float) + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(local_softmax_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)prm.BH * p.T * prm.qtiles;
  const int grid = (int)(units < sms ? units : sms);
  local_softmax_tc_kernel<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
