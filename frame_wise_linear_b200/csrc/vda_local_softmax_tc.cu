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
// Design (persistent, one CTA per SM, 6 warps), work unit = 128 query tokens
// of one frame of one head; its key tiles are 128 tokens of one key frame (the
// last tile of a frame partial) and then of the text:
//   warp 0     TMA producer: the unit's Q tile, then K and V tiles through a
//              2-stage ring (64 KB a stage).
//   warp 1     TMEM and the MMAs: S_j = Q K_j^T into one of two 128-column
//              score buffers, issued one tile ahead, and O += P_j V_j into a
//              128-column accumulator once the softmax has written P_j.
//   warps 2..5 softmax, one thread per query row: the row's scores from TMEM,
//              the running maximum and sum (log2 domain), P_j = exp2 of the
//              scaled scores as bf16 into shared memory; the accumulator is
//              rescaled only when the maximum grows by more than 2^8 (the
//              exponentials with a stale maximum stay below 2^8, and O and
//              the sum share that maximum, so the quotient is exact).  After
//              the last tile: O / sum, times sigmoid(G), stored from
//              registers as whole 128-byte row segments (8-lane transpose).
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"
#include "vda_tok.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kRows = 128;                   // query and key tokens per tile
constexpr int kBox = kRows * 64 * 2;         // 128 rows x 64 features bf16: 16 KB
constexpr int kTile = 2 * kBox;              // 32 KB
constexpr int kBlock = 5;                    // frames per block of the window
constexpr float kRescale = 8.f;              // log2 growth of the maximum that forces a rescale
constexpr uint32_t kTmemCols = 512;          // S0 | S1 | O
constexpr uint32_t kOCol = 256;
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
  uint64_t kv_full[2], kv_empty[2];
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
  uint8_t* kvbuf = base + kTile;             // 2 stages: K tile | V tile
  uint8_t* pbuf = kvbuf + 4 * kTile;         // 2 P tiles
  Shared& sh = *reinterpret_cast<Shared*>(pbuf + 2 * kTile);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int units = p.BH * p.T * p.qtiles;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    mbar_init(&sh.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.kv_full[i], 1);
      mbar_init(&sh.kv_empty[i], 1);
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.s_free[i], 128);
      mbar_init(&sh.p_full[i], 128);
      mbar_init(&sh.pv_done[i], 1);
    }
    mbar_init(&sh.o_free, 128);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_q = policy_evict_first();
      const uint64_t pol_kv = policy_evict_last();   // a key frame serves 15 query frames
      int kv_issued = 0, q_issued = 0, it = 0, ui = 0;
      bool ok = true;
      for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
        const int qt = w % p.qtiles, t = (w / p.qtiles) % p.T, bh = w / (p.qtiles * p.T);
        const TokPos qpos = tok_pos(p.g, bh * p.T + t, false);
        if (!(ok = mbar_wait(&sh.q_empty, (ui & 1) ^ 1))) break;   // the previous unit's S MMAs are done
        mbar_expect_tx(&sh.q_full, kTile);
        tok_load(qbuf, &p.mQ, &sh.q_full, p.g, qpos, 0, qt * kRows, pol_q);
        tok_load(qbuf + kBox, &p.mQ, &sh.q_full, p.g, qpos, 64, qt * kRows, pol_q);
        ++q_issued;
        const KeyFrames kf = key_frames(t, p.T);
        const int J = key_tiles(p, kf);
        int cur = -2;
        TokPos kpos{};
        for (int j = 0; j < J; ++j, ++it) {
          const int s = it & 1;
          if (!(ok = mbar_wait(&sh.kv_empty[s], ((it >> 1) & 1) ^ 1))) break;
          const KeyTile kt = key_tile(p, kf, j);
          if (kt.frame != cur) {
            kpos = kt.text ? tok_pos(p.g, bh, true) : tok_pos(p.g, bh * p.T + kt.frame, false);
            cur = kt.frame;
          }
          const CUtensorMap* mk = kt.text ? &p.mKt : &p.mK;
          const CUtensorMap* mv = kt.text ? &p.mVt : &p.mV;
          uint8_t* st = kvbuf + s * 2 * kTile;
          mbar_expect_tx(&sh.kv_full[s], 2 * kTile);
          tok_load(st, mk, &sh.kv_full[s], p.g, kpos, 0, kt.y, pol_kv);
          tok_load(st + kBox, mk, &sh.kv_full[s], p.g, kpos, 64, kt.y, pol_kv);
          tok_load(st + kTile, mv, &sh.kv_full[s], p.g, kpos, 0, kt.y, pol_kv);
          tok_load(st + kTile + kBox, mv, &sh.kv_full[s], p.g, kpos, 64, kt.y, pol_kv);
          ++kv_issued;
        }
      }
      if (!ok) set_abort(sh, p.err);
      if (aborted(sh)) {   // the loads still in flight land before exit
        for (int c = kv_issued > 2 ? kv_issued - 2 : 0; c < kv_issued; ++c)
          mbar_wait(&sh.kv_full[c & 1], (c >> 1) & 1);
        if (q_issued > 0) mbar_wait(&sh.q_full, (q_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMAs
    if (lane == 0) {
      const uint32_t qa = smem_u32(qbuf), kva = smem_u32(kvbuf), pa = smem_u32(pbuf);
      int it = 0, ui = 0;   // global tile counter (ring and S / P buffers), unit counter
      bool ok = true;
      // S = Q K^T for the tile at ring position `pos` into S buffer pos & 1.
      auto issue_s = [&](int pos) -> bool {
        const int s = pos & 1;
        if (!mbar_wait(&sh.s_free[s], ((pos >> 1) & 1) ^ 1)) return false;   // the softmax has read it
        if (!mbar_wait(&sh.kv_full[s], (pos >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t ka = kva + s * 2 * kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k / 4) * kBox + (k % 4) * 32;
          mma_bf16_ss(tmem + s * 128, smem_desc(qa + off, 16, 1024, kSwizzle128B),
                      smem_desc(ka + off, 16, 1024, kSwizzle128B), kIdescS, k ? 1u : 0u);
        }
        mma_commit(&sh.s_full[s]);
        return true;
      };
      for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
        const int t = (w / p.qtiles) % p.T;
        const int J = key_tiles(p, key_frames(t, p.T));
        if (!(ok = mbar_wait(&sh.q_full, ui & 1))) break;
        if (!(ok = issue_s(it))) break;
        for (int j = 0; j < J && ok; ++j) {
          const int pos = it + j, s = pos & 1;
          if (j + 1 < J && !(ok = issue_s(pos + 1))) break;
          if (j + 1 == J) mma_commit(&sh.q_empty);   // the unit's last S MMAs read Q before anything after
          if (j == 0 && !(ok = mbar_wait(&sh.o_free, (ui & 1) ^ 1))) break;   // the previous unit's O is read
          if (!(ok = mbar_wait(&sh.p_full[s], (pos >> 1) & 1))) break;
          tc_fence_after();
          const uint32_t va = kva + s * 2 * kTile + kTile, pb = pa + s * kTile;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            mma_bf16_ss(tmem + kOCol, smem_desc(pb + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B),
                        smem_desc(va + k * 16 * 128, kBox, 1024, kSwizzle128B), kIdescO, (j | k) ? 1u : 0u);
          }
          mma_commit(&sh.pv_done[s]);
          mma_commit(&sh.kv_empty[s]);
        }
        it += J;
      }
      if (!ok) set_abort(sh, p.err);
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int row = (warp % 4) * 32 + lane;   // query row = TMEM lane
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;
    const size_t rstride = tok_row_stride(p.g);
    int it = 0, ui = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < units && ok; w += gridDim.x, ++ui) {
      const int qt = w % p.qtiles, t = (w / p.qtiles) % p.T, bh = w / (p.qtiles * p.T);
      const KeyFrames kf = key_frames(t, p.T);
      const int J = key_tiles(p, kf);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < J; ++j) {
        const int pos = it + j, s = pos & 1;
        const KeyTile kt = key_tile(p, kf, j);
        const bool stall = p.stall == VDA_TEST_STALL_SOFTMAX && blockIdx.x == 0 && pos == 0;
        if (!(ok = !aborted(sh) && mbar_wait_or_stall(&sh.s_full[s], (pos >> 1) & 1, &sh.never, stall))) break;
        tc_fence_after();
        float x[128];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + s * 128 + lane_off + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(r[e]);
        }
        tc_fence_before();
        mbar_arrive(&sh.s_free[s]);            // the MMAs may write the next scores here
        float mt = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; ++e) {
          x[e] = e < kt.valid ? x[e] * p.c : -INFINITY;   // scores in log2 units; rows past the keys excluded
          mt = fmaxf(mt, x[e]);
        }
        // P_j's buffer is free once PV_{j-2} is done, and a rescale of O needs PV_{j-1} done.
        const bool grow = j == 0 || mt > m + kRescale;
        if (j >= 2 && !(ok = mbar_wait(&sh.pv_done[s], ((pos - 2) >> 1) & 1))) break;
        if (grow) {
          const float mn = fmaxf(m, mt);
          if (j >= 1) {
            if (!(ok = mbar_wait(&sh.pv_done[s ^ 1], ((pos - 1) >> 1) & 1))) break;
            tc_fence_after();
            const float a = ex2(m - mn);
            l *= a;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t r[32];
              tmem_ld_32x32b_x32(tmem + kOCol + lane_off + c * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(a * __uint_as_float(r[e]));
              tmem_st_32x32b_x32(tmem + kOCol + lane_off + c * 32, r);
            }
            tmem_st_wait();
          }
          m = mn;
        }
        uint8_t* pt = pbuf + s * kTile;
#pragma unroll
        for (int c = 0; c < 16; ++c) {           // keys 8c .. 8c + 7
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[e] = ex2(x[8 * c + e] - m);
            l += v[e];
          }
          *reinterpret_cast<uint4*>(pt + (c >> 3) * kBox + sw128(row, c & 7)) =
              make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.p_full[s]);
      }
      if (!ok) break;
      // ---- epilogue: O / l times sigmoid(G), rows past n skipped
      const int last = it + J - 1;
      if (!(ok = !aborted(sh) && mbar_wait(&sh.pv_done[last & 1], (last >> 1) & 1))) break;
      tc_fence_after();
      const TokPos qpos = tok_pos(p.g, bh * p.T + t, false);
      const size_t obase = tok_base(p.g, qpos, p.n, false);
      const int tok = qt * kRows + row;
      const float inv = 1.f / l;
      const int r0 = (warp % 4) * 32 + 8 * (lane >> 3);
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {          // 64 columns at a time
        uint4 ch[8];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + kOCol + lane_off + hf * 64 + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = hf * 64 + c * 32 + q * 8;
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
        if (hf == 1) {
          tc_fence_before();
          mbar_arrive(&sh.o_free);               // the next unit's first PV may overwrite O
        }
        transpose8(ch, lane & 7);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int tr = qt * kRows + r0 + k;
          if (tr < p.n) *reinterpret_cast<uint4*>(p.O + obase + (size_t)tr * rstride + hf * 64 + (lane & 7) * 8) = ch[k];
        }
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
  const size_t smem = 1024 + 7 * kTile + sizeof(Shared);
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
