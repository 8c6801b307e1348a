// Backward of the Gram products on tcgen05 tensor cores.  A_t = K_t^T K_t +
// lambda I and B_t = K_t^T V_t ("VDN-MiniMax-H3" (aiezz.com), section 03,
// normal-equation item) give, for gradients dA_t and dB_t of a unit (a frame,
// or a head's text):
//     dK = K (dA + dA^T) + V dB^T,      dV = K dB,
// with W1 = dA + dA^T and dB as bf16 operands ([units][256][128]: W1 rows,
// then dB rows), bf16 K, V, dK, dV; d = 128.
//
// Per 128-token tile the MMAs accumulate dK = K W1 (B = W1, symmetric, read
// K-major) + V dB^T (B = dB read K-major) and dV = K dB (B = dB read
// MN-major: the same shared-memory image of dB both ways) into a TMEM buffer
// pair; the epilogue stores both through a staging box per column half (TMA
// stores, rows past the unit's token count clipped), so a K / V stage is free
// as soon as its MMAs are done.
//
// Design (persistent, one CTA per SM, 10 warps), work = 128-row tiles of the
// frames and then of the text, a contiguous range of tiles per CTA:
//   warp 0     TMA producer: W1 | dB per unit, K and V tiles (2 stages).
//   warp 1     TMEM (2 x (128 + 128) columns) and the MMAs (one thread).
//   warps 2..9 epilogue: two warps per TMEM lane quarter, each on 64 of the
//              128 columns of dK and of dV.
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
constexpr int kStages = 2;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescK = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ false);   // K W1, V dB^T
constexpr uint32_t kIdescV = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ true);    // K dB

struct GramBwdParams {
  CUtensorMap mK, mV, mW;         // frames: [frames][n][128], W [frames][256][128]
  CUtensorMap mKt, mVt, mWt;      // text: [heads][n_txt][128], W [heads][256][128]
  CUtensorMap mdK, mdV, mdKt, mdVt;   // the outputs, same shapes as K, V, K_txt, V_txt
  const __nv_bfloat16* W;
  const __nv_bfloat16* Wt;
  unsigned* err;
  int frames, heads, n, n_txt;
  int tpf, tpt;                   // tiles per frame, per text unit
  TokGeom g;                      // the layout of K, V, dK, dV and the text's
  int stall;                      // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t d_full[2], t_empty[2];
  uint64_t w_full, w_empty;
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

// Tile t of the sequence: its unit (frames first, then the text's heads), the
// first token row, and whether the unit is text.
struct TileRef {
  int unit;    // global unit index: frame, or frames + head
  int item;    // frame or head
  int y;
  bool text;
};
__device__ __forceinline__ TileRef tile_ref(const GramBwdParams& p, int t) {
  const int ft = p.frames * p.tpf;
  if (t < ft) return TileRef{t / p.tpf, t / p.tpf, (t % p.tpf) * kRows, false};
  const int r = t - ft;
  return TileRef{p.frames + r / p.tpt, r / p.tpt, (r % p.tpt) * kRows, true};
}

__global__ void __launch_bounds__(kThreads, 1) gram_bwd_tc_kernel(const __grid_constant__ GramBwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* wbuf = base;                             // W1 (32 KB) | dB (32 KB)
  uint8_t* kvbuf = wbuf + 2 * kTile;                // kStages x (K tile | V tile)
  uint8_t* stg = kvbuf + kStages * 2 * kTile;       // output staging: one 64-column box per half
  Shared& sh = *reinterpret_cast<Shared*>(stg + kTile);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const long long total = (long long)p.frames * p.tpf + (long long)p.heads * p.tpt;
  const int t_begin = (int)(total * blockIdx.x / gridDim.x);
  const int t_end = (int)(total * (blockIdx.x + 1) / gridDim.x);
  const int J = t_end - t_begin;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sh.kv_full[i], 1);
      mbar_init(&sh.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.d_full[i], 1);
      mbar_init(&sh.t_empty[i], 256);
    }
    mbar_init(&sh.w_full, 1);
    mbar_init(&sh.w_empty, 1);
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
    tma_prefetch_desc(&p.mK);
    tma_prefetch_desc(&p.mV);
    tma_prefetch_desc(&p.mW);
    if (p.heads > 0 && p.tpt > 0) {
      tma_prefetch_desc(&p.mKt);
      tma_prefetch_desc(&p.mVt);
      tma_prefetch_desc(&p.mWt);
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
      int kv_issued = 0, w_issued = 0, cur = -1, pos_unit = -1;
      TokPos q{};
      for (int j = 0; j < J; ++j) {
        const TileRef r = tile_ref(p, t_begin + j);
        if (r.unit != pos_unit) {
          q = tok_pos(p.g, r.item, r.text);
          pos_unit = r.unit;
        }
        const int st = j & 1;
        if (!mbar_wait(&sh.kv_empty[st], ((j >> 1) & 1) ^ 1)) { set_abort(sh, p.err); break; }
        uint8_t* kv = kvbuf + st * 2 * kTile;
        const CUtensorMap* mk = r.text ? &p.mKt : &p.mK;
        const CUtensorMap* mv = r.text ? &p.mVt : &p.mV;
        mbar_expect_tx(&sh.kv_full[st], 2 * kTile);
        tok_load(kv, mk, &sh.kv_full[st], p.g, q, 0, r.y, pol);
        tok_load(kv + kBox, mk, &sh.kv_full[st], p.g, q, 64, r.y, pol);
        tok_load(kv + kTile, mv, &sh.kv_full[st], p.g, q, 0, r.y, pol);
        tok_load(kv + kTile + kBox, mv, &sh.kv_full[st], p.g, q, 64, r.y, pol);
        ++kv_issued;
        if (r.unit != cur) {
          // The unit's W1 | dB, once the previous unit's MMAs are done with the buffer.
          if (w_issued > 0 && !mbar_wait(&sh.w_empty, (w_issued - 1) & 1)) { set_abort(sh, p.err); break; }
          const CUtensorMap* mw = r.text ? &p.mWt : &p.mW;
          mbar_expect_tx(&sh.w_full, 2 * kTile);
#pragma unroll
          for (int b = 0; b < 4; ++b)
            tma_load_3d(wbuf + b * kBox, mw, &sh.w_full, 64 * (b & 1), 128 * (b >> 1), r.item, pol);
          ++w_issued;
          cur = r.unit;
          // The next unit's operands into L2 while this one's tiles run.
          const int nxt = r.item + 1;
          if (!r.text && nxt < p.frames) bulk_prefetch_l2(p.W + (size_t)nxt * 256 * 128, 256 * 128 * 2);
          if (r.text && nxt < p.heads) bulk_prefetch_l2(p.Wt + (size_t)nxt * 256 * 128, 256 * 128 * 2);
        }
      }
      if (aborted(sh)) {  // let the loads still in flight land before exit
        for (int c = kv_issued > kStages ? kv_issued - kStages : 0; c < kv_issued; ++c)
          mbar_wait(&sh.kv_full[c & 1], (c >> 1) & 1);
        if (w_issued > 0) mbar_wait(&sh.w_full, (w_issued - 1) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t w1 = smem_u32(wbuf), db = w1 + kTile;
      const uint32_t kvaddr = smem_u32(kvbuf);
      int cur = -1, units = 0;
      bool ok = true;
      for (int j = 0; j < J && ok; ++j) {
        const TileRef r = tile_ref(p, t_begin + j);
        const int st = j & 1, tb = j & 1;
        if (r.unit != cur) {
          if (!(ok = mbar_wait(&sh.w_full, units & 1))) break;
          ++units;
          cur = r.unit;
        }
        if (!(ok = mbar_wait(&sh.t_empty[tb], ((j >> 1) & 1) ^ 1))) break;
        const bool stall = p.stall == VDA_TEST_STALL_GBWD_TILE && blockIdx.x == 0 && j == 0;
        if (!(ok = mbar_wait_or_stall(&sh.kv_full[st], (j >> 1) & 1, &sh.never, stall))) break;
        tc_fence_after();
        const uint32_t ka = kvaddr + st * 2 * kTile, va = ka + kTile;
        const uint32_t dk = tmem + tb * 256, dv = dk + 128;
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // dK = K W1
          const uint64_t a = smem_desc(ka + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(w1 + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          mma_bf16_ss(dk, a, b, kIdescK, k ? 1u : 0u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // dK += V dB^T
          const uint64_t a = smem_desc(va + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(db + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          mma_bf16_ss(dk, a, b, kIdescK, 1u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {   // dV = K dB
          const uint64_t a = smem_desc(ka + (k / 4) * kBox + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(db + k * 16 * 128, kBox, 1024, kSwizzle128B);
          mma_bf16_ss(dv, a, b, kIdescV, k ? 1u : 0u);
        }
        mma_commit(&sh.kv_empty[st]);
        mma_commit(&sh.d_full[tb]);
        const bool last_of_unit = (j + 1 == J) || tile_ref(p, t_begin + j + 1).unit != r.unit;
        if (last_of_unit) mma_commit(&sh.w_empty);
      }
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
    for (int j = 0; j < J; ++j) {
      const TileRef r = tile_ref(p, t_begin + j);
      const int tb = j & 1;
      const bool stall = p.stall == VDA_TEST_STALL_GBWD_STORE && blockIdx.x == 0 && j == 1;
      bool ok = !aborted(sh) && mbar_wait_or_stall(&sh.d_full[tb], (j >> 1) & 1, &sh.never, stall);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(1 + half, 128, !ok)) break;   // one decision per half
      tc_fence_after();
      uint8_t* box = stg + half * kBox;
      const TokPos q = et % 128 == 0 ? tok_pos(p.g, r.item, r.text) : TokPos{};   // the storing thread's
#pragma unroll 1
      for (int m = 0; m < 2; ++m) {           // dK, then dV
        const uint32_t taddr = tmem + tb * 256 + m * 128 + half * 64 + lane_off;
        // The staging box is free once the half's previous store has read it.
        if (et % 128 == 0) bulk_wait_read<0>();
        named_bar_sync(1 + half, 128);
#pragma unroll 1
        for (int c = 0; c < 2; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<uint4*>(box + sw128(row, c * 4 + q)) =
                make_uint4(pack_bf16(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                           pack_bf16(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                           pack_bf16(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                           pack_bf16(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
        }
        fence_proxy_async_smem();
        named_bar_sync(1 + half, 128);
        if (et % 128 == 0) {   // rows past the unit's token count are clipped by the TMA
          const CUtensorMap* map = m == 0 ? (r.text ? &p.mdKt : &p.mdK) : (r.text ? &p.mdVt : &p.mdV);
          tok_store(map, box, p.g, q, 64 * half, r.y);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.t_empty[tb]);
    }
    if (et % 128 == 0) bulk_wait<0>();         // the stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_gram_bwd_tc(const vda_problem& p, const __nv_bfloat16* K, const __nv_bfloat16* V,
                               const __nv_bfloat16* W, const __nv_bfloat16* Kt, const __nv_bfloat16* Vt,
                               const __nv_bfloat16* Wt, __nv_bfloat16* dK, __nv_bfloat16* dV, __nv_bfloat16* dKt,
                               __nv_bfloat16* dVt, unsigned* err, cudaStream_t st) {
  GramBwdParams prm;
  memset(&prm, 0, sizeof(prm));
  const int heads = p.B * p.H, frames = heads * p.T;
  if (!make_tok_map(&prm.mK, K, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mV, V, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_bf16_rows_map(&prm.mW, W, 256, frames, 128))
    return cudaErrorInvalidValue;
  if (!make_tok_map(&prm.mdK, dK, p.layout, p.B, p.H, p.T, p.n, kRows) ||
      !make_tok_map(&prm.mdV, dV, p.layout, p.B, p.H, p.T, p.n, kRows))
    return cudaErrorInvalidValue;
  const bool text = p.n_txt > 0;
  if (text && (!make_tok_map(&prm.mKt, Kt, p.layout, p.B, p.H, 1, p.n_txt, kRows) ||
               !make_tok_map(&prm.mVt, Vt, p.layout, p.B, p.H, 1, p.n_txt, kRows) ||
               !make_bf16_rows_map(&prm.mWt, Wt, 256, heads, 128) ||
               !make_tok_map(&prm.mdKt, dKt, p.layout, p.B, p.H, 1, p.n_txt, kRows) ||
               !make_tok_map(&prm.mdVt, dVt, p.layout, p.B, p.H, 1, p.n_txt, kRows)))
    return cudaErrorInvalidValue;
  prm.W = W;
  prm.Wt = Wt;
  prm.err = err;
  prm.frames = frames;
  prm.heads = text ? heads : 0;
  prm.n = p.n;
  prm.n_txt = p.n_txt;
  prm.tpf = (p.n + kRows - 1) / kRows;
  prm.tpt = text ? (p.n_txt + kRows - 1) / kRows : 0;
  prm.g = TokGeom{p.layout, p.H, p.T};
  prm.stall = p.test_stall;
  const size_t smem = 1024 + (3 + 2 * kStages) * kTile + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(gram_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = (long long)frames * prm.tpf + (long long)prm.heads * prm.tpt;
  const int grid = (int)(tiles < sms ? tiles : sms);
  gram_bwd_tc_kernel<<<grid, kThreads, smem, st>>>(prm);
  return cudaGetLastError();
}

}  // namespace vda
