// The backward's 128 x 128 steps between its two streaming kernels, on
// tcgen05 tensor cores: the operands of the Gram products' backward, per
// frame and per head's text.
//
// With the forward read as "VDN-MiniMax-H3" (aiezz.com), section 03 states it
// (a normal-equation solve per frame, the text written once into both
// directional states), the gradients of A_t = K_t^T K_t + lambda I and
// B_t = K_t^T V_t are, for the adjoints Gf_t, Gb_t of the two scans and the
// states S^f_t, S^b_t,
//     dA_t = -(Gf_t S^f_t^T + Gb_t S^b_t^T),     dB_t = Gf_t + Gb_t,
// and the Gram backward needs W1 = dA + dA^T and dB.  So, per frame,
//     W1 = -(Gf S^f^T + S^f Gf^T + Gb S^b^T + S^b Gb^T)
// is four products of bf16 128 x 128 operands, all K-major (row-major
// storage), accumulated in TMEM; dB is an element-wise sum.  For a head's
// text (slot 0), with M_0 = lambda A_0^{-1}, X_0 = Gf_1 + Gb_T and B_0:
//     G_0 = M_0 X_0,   S_0 = M_0 B_0 / lambda,   dB_0 = G_0,
//     W1_0 = -(G_0 S_0^T + S_0 G_0^T).
//
// Design (persistent, one CTA per SM, 6 warps):
//   text first: the CTAs take the heads round-robin.  M_0 (the scan's bf16
//     hi | lo operand image) arrives by bulk copy; the four epilogue warps
//     (one thread per row) build [X_0 | B_0 / lambda] as a bf16 hi / lo
//     MN-major operand; 24 MMAs (M = 128, N = 256, three passes hi hi, hi lo,
//     lo hi) give G_0 | S_0 in TMEM; the rows of G_0 and S_0 go back to
//     shared memory as hi / lo K-major images, and 48 MMAs (K = 256: G_0 S_0^T
//     and S_0 G_0^T, three passes) give W1_0.  The text's rows are stored from
//     registers.
//   frames next, a contiguous range per CTA (a CTA that ran a text chain
//   takes about 8 frames fewer):
//     warp 0     TMA producer: per frame two half-units, (Gf, S^f) and then
//                (Gb, S^b), 64 KB each, through a 2-slot ring.
//     warp 1     TMEM and the 32 MMAs of a frame (16 per half-unit) into one
//                of two 128-column accumulators.
//     warps 2..5 epilogue: W1 = -acc and dB = Gf + Gb (the bf16 adjoints, read
//                from global memory, where the producer's loads have just
//                brought them into L2, before the wait for the frame's MMAs)
//                through two 32 KB staging boxes, TMA stores into the
//                [frames][256][128] operand image.
// Every wait is bounded; a wait that runs out sets the timeout bit of the
// error word and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kBox = 128 * 64 * 2;           // 128 rows x 64 columns bf16: 16 KB
constexpr int kMat = 2 * kBox;               // one 128 x 128 bf16 operand image: 32 KB
constexpr int kSlot = 2 * kMat;              // a half-unit: an adjoint and a state
constexpr int kStage = 2 * kSlot;            // the ring, 128 KB
constexpr int kEpiBar = 1;                   // named barrier of the epilogue warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kIdescKK = idesc_bf16_f32(128, 128, /*a MN*/ false, /*b MN*/ false);
constexpr uint32_t kIdescText = idesc_bf16_f32(128, 256, /*a MN*/ false, /*b MN*/ true);

struct BwdOperandsParams {
  CUtensorMap mGf, mSf, mGb, mSb;   // [frames][128][128] bf16, 64-column x 128-row boxes
  CUtensorMap mW;                   // [frames][256][128] bf16 (W1 rows, then dB rows), same boxes
  const __nv_bfloat16* Gf;          // the adjoints, bf16, [frames][128][128]
  const __nv_bfloat16* Gb;
  const uint8_t* M;                 // per slot 64 KB: M hi | M lo (the scan's operand image)
  const float* Bm;                  // per slot B_t, 128 x 128 float
  __nv_bfloat16* Wt;                // [heads][256][128] bf16: the text's W1_0 | dB_0 (NULL: no text)
  unsigned* err;
  int frames, heads, T;
  int text_weight;                  // frames a head's text chain counts for in the frame split
  float inv_lam;
  int stall;                        // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t full[2], empty[2];
  uint64_t t_full[2], t_empty[2];
  uint64_t m_full, x_done, w_done;
  uint64_t drain;
  uint64_t never;                   // testing hook: nothing arrives on it
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

// x split into bf16 hi + lo (hi = x rounded, lo = the rest rounded).
__device__ __forceinline__ void split(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = x - hi;
}

// Eight floats of bf16 as one 16-byte chunk.
__device__ __forceinline__ uint4 pack8(const float (&v)[8]) {
  return make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
}

// Row `row`, columns 8c .. 8c + 7 of a 128 x 128 K-major image (two boxes of
// 64 columns, 128-byte swizzle): byte offset.
__device__ __forceinline__ uint32_t kimg(int row, int c) { return (c >> 3) * kBox + sw128(row, c & 7); }

__global__ void __launch_bounds__(kThreads, 1) bwd_operands_tc_kernel(const __grid_constant__ BwdOperandsParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = base;                     // frames: 2 slots of 64 KB; text: M_0, then G_0 / S_0 images
  uint8_t* stg = base + kStage;             // frames: W1 and dB staging; text: [X_0 | B_0/lambda] hi
  Shared& sh = *reinterpret_cast<Shared*>(base + kStage + 2 * kMat);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const bool epi = warp >= 2;
  const int row = (warp % 4) * 32 + lane;   // epilogue: TMEM lane = matrix row
  const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
      mbar_init(&sh.t_full[i], 1);
      mbar_init(&sh.t_empty[i], 128);
    }
    mbar_init(&sh.m_full, 1);
    mbar_init(&sh.x_done, 1);
    mbar_init(&sh.w_done, 1);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.never, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  // The adjoints come from the kernel before this one.
  griddep_wait();

  // ---------------------------------------------------------------- text
  // Straight-line phases separated by __syncthreads (every thread passes
  // every one); a wait that runs out sets the abort flag and the phases
  // still run to the end on whatever is in shared memory.
  int text_units = 0;
  for (int bh = blockIdx.x; p.Wt && bh < p.heads; bh += gridDim.x, ++text_units) {
    const int ph = text_units & 1;
    uint8_t* mimg = ring;                   // 64 KB: M_0 hi | lo
    uint8_t* xb_hi = ring + 65536;          // [X_0 | B_0 / lambda], MN-major, 4 blocks of 64 columns
    uint8_t* xb_lo = stg;
    if (threadIdx.x == 0) {
      mbar_expect_tx(&sh.m_full, 65536);
      const uint8_t* src = p.M + (size_t)bh * (p.T + 1) * 65536;   // the head's text slot
      bulk_load(mimg, src, 32768, &sh.m_full);
      bulk_load(mimg + 32768, src + 32768, 32768, &sh.m_full);
    }
    if (epi) {
      // row k of X_0 = Gf_1 + Gb_T (frames 1 and T of the head) and of B_0 / lambda
      const __nv_bfloat16* gf1 = p.Gf + ((size_t)bh * p.T + 0) * 128 * 128 + (size_t)row * 128;
      const __nv_bfloat16* gbT = p.Gb + ((size_t)bh * p.T + (p.T - 1)) * 128 * 128 + (size_t)row * 128;
      const float* b0 = p.Bm + (size_t)bh * (p.T + 1) * 128 * 128 + (size_t)row * 128;
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {          // columns 8c .. 8c + 7
        const uint4 f = *reinterpret_cast<const uint4*>(gf1 + 8 * c);
        const uint4 g = *reinterpret_cast<const uint4*>(gbT + 8 * c);
        const __nv_bfloat162* f2 = reinterpret_cast<const __nv_bfloat162*>(&f);
        const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
        const float4 bA = *reinterpret_cast<const float4*>(b0 + 8 * c);
        const float4 bB = *reinterpret_cast<const float4*>(b0 + 8 * c + 4);
        const float bv[8] = {bA.x, bA.y, bA.z, bA.w, bB.x, bB.y, bB.z, bB.w};
        float xh[8], xl[8], bh8[8], bl8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 a = __bfloat1622float2(f2[e]), b = __bfloat1622float2(g2[e]);
          split(a.x + b.x, xh[2 * e], xl[2 * e]);
          split(a.y + b.y, xh[2 * e + 1], xl[2 * e + 1]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) split(bv[e] * p.inv_lam, bh8[e], bl8[e]);
        // MN-major image: block (column / 64), row k, chunk (column % 64) / 8
        const uint32_t ox = (c >> 3) * 16384u + sw128(row, c & 7);
        const uint32_t ob = (2 + (c >> 3)) * 16384u + sw128(row, c & 7);
        *reinterpret_cast<uint4*>(xb_hi + ox) = pack8(xh);
        *reinterpret_cast<uint4*>(xb_lo + ox) = pack8(xl);
        *reinterpret_cast<uint4*>(xb_hi + ob) = pack8(bh8);
        *reinterpret_cast<uint4*>(xb_lo + ob) = pack8(bl8);
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 32) {                  // warp 1: G_0 | S_0 = M_0 [X_0 | B_0 / lambda]
      if (!mbar_wait(&sh.m_full, ph)) set_abort(sh, p.err);
      tc_fence_after();
      const uint32_t ma = smem_u32(mimg), xh = smem_u32(xb_hi), xl = smem_u32(xb_lo);
#pragma unroll
      for (int pass = 0; pass < 3; ++pass) {  // M_hi X_hi, M_hi X_lo, M_lo X_hi
        const uint32_t a0 = ma + (pass == 2 ? 32768u : 0u);
        const uint32_t b0 = pass == 1 ? xl : xh;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint64_t a = smem_desc(a0 + (k / 4) * 16384 + (k % 4) * 32, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(b0 + k * 16 * 128, 16384, 1024, kSwizzle128B);
          mma_bf16_ss(tmem, a, b, kIdescText, (pass | k) ? 1u : 0u);
        }
      }
      mma_commit(&sh.x_done);
    }
    if (epi) {
      if (!mbar_wait(&sh.x_done, ph)) set_abort(sh, p.err);
      tc_fence_after();
    }
    __syncthreads();                          // the MMAs are done with M_0 and [X_0 | B_0]
    // G_0 and S_0 rows as hi / lo K-major images (32 KB each) in the ring;
    // dB_0 = G_0 straight to the text's operand image.
    uint8_t* g_hi = ring;
    uint8_t* g_lo = ring + kMat;
    uint8_t* s_hi = ring + 2 * kMat;
    uint8_t* s_lo = ring + 3 * kMat;
    if (epi) {
      __nv_bfloat16* db = p.Wt + ((size_t)bh * 256 + 128 + row) * 128;
#pragma unroll 1
      for (int q = 0; q < 8; ++q) {           // 32 columns of G_0 (q < 4) or S_0 (q >= 4)
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_off + q * 32, r);
        tmem_ld_wait();
        uint8_t* hi = q < 4 ? g_hi : s_hi;
        uint8_t* lo = q < 4 ? g_lo : s_lo;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float h[8], l[8], v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[e] = __uint_as_float(r[8 * j + e]);
            split(v[e], h[e], l[e]);
          }
          const int c = (q % 4) * 4 + j;      // 8-column chunk of the 128
          *reinterpret_cast<uint4*>(hi + kimg(row, c)) = pack8(h);
          *reinterpret_cast<uint4*>(lo + kimg(row, c)) = pack8(l);
          if (q < 4) *reinterpret_cast<uint4*>(db + 8 * c) = pack8(v);
        }
      }
      fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 32) {                  // W1_0 accumulator: columns 256..383
      tc_fence_after();
      const uint32_t gh = smem_u32(g_hi), gl = smem_u32(g_lo), shh = smem_u32(s_hi), sl = smem_u32(s_lo);
#pragma unroll
      for (int pass = 0; pass < 3; ++pass) {  // hi hi, hi lo, lo hi
#pragma unroll
        for (int k = 0; k < 16; ++k) {        // K = 256: [G_0 | S_0] times [S_0 | G_0]^T
          const bool first = k < 8;
          const uint32_t ab = first ? (pass == 2 ? gl : gh) : (pass == 2 ? sl : shh);
          const uint32_t bb = first ? (pass == 1 ? sl : shh) : (pass == 1 ? gl : gh);
          const uint32_t off = ((k % 8) / 4) * kBox + (k % 4) * 32;
          const uint64_t a = smem_desc(ab + off, 16, 1024, kSwizzle128B);
          const uint64_t b = smem_desc(bb + off, 16, 1024, kSwizzle128B);
          mma_bf16_ss(tmem + 256, a, b, kIdescKK, (pass | k) ? 1u : 0u);
        }
      }
      mma_commit(&sh.w_done);
    }
    if (epi) {
      if (!mbar_wait(&sh.w_done, ph)) set_abort(sh, p.err);
      tc_fence_after();
      __nv_bfloat16* w1 = p.Wt + ((size_t)bh * 256 + row) * 128;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + lane_off + 256 + q * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = -__uint_as_float(r[8 * j + e]);
          *reinterpret_cast<uint4*>(w1 + 8 * (q * 4 + j)) = pack8(v);
        }
      }
    }
    tc_fence_before();
    __syncthreads();                          // the ring and TMEM are free again
    tc_fence_after();
  }

  // ---------------------------------------------------------------- frames
  // Contiguous frame ranges, with each text chain counted as text_weight
  // frames of its CTA's share (the CTAs that ran a text chain take fewer
  // frames).  Split points b(c) = V(c) - w * texts(< c), V(c) = total c / grid:
  // b(0) = 0, b(grid) = frames, and the host keeps b non-decreasing.
  auto split = [&](int c) -> int {
    const long long w = p.Wt ? p.text_weight : 0;
    const long long total = p.frames + w * p.heads;
    const long long texts = min((long long)c, (long long)p.heads);   // heads of the CTAs before c (one each)
    return (int)(total * c / gridDim.x - w * texts);
  };
  const int f_begin = split(blockIdx.x);
  const int f_end = split(blockIdx.x + 1);
  const int J = f_end - f_begin;
  if (warp == 0) {
    if (lane == 0 && !aborted(sh)) {
      const uint64_t pol = policy_evict_last();   // the epilogue reads the adjoints again
      int issued = 0;
      for (int j = 0; j < 2 * J; ++j) {       // half-unit j: frame f_begin + j / 2, part j % 2
        const int s = j & 1;
        if (!mbar_wait(&sh.empty[s], ((j >> 1) & 1) ^ 1)) {
          set_abort(sh, p.err);
          break;
        }
        const int f = f_begin + j / 2;
        const CUtensorMap* mg = s == 0 ? &p.mGf : &p.mGb;
        const CUtensorMap* ms = s == 0 ? &p.mSf : &p.mSb;
        uint8_t* dst = ring + s * kSlot;
        mbar_expect_tx(&sh.full[s], kSlot);
        tma_load_3d(dst, mg, &sh.full[s], 0, 0, f, pol);
        tma_load_3d(dst + kBox, mg, &sh.full[s], 64, 0, f, pol);
        tma_load_3d(dst + kMat, ms, &sh.full[s], 0, 0, f, pol);
        tma_load_3d(dst + kMat + kBox, ms, &sh.full[s], 64, 0, f, pol);
        ++issued;
      }
      if (aborted(sh))   // the loads still in flight land before exit
        for (int c = issued > 2 ? issued - 2 : 0; c < issued; ++c) mbar_wait(&sh.full[c & 1], (c >> 1) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = !aborted(sh);
      for (int j = 0; j < J && ok; ++j) {
        const int tb = j & 1;
        if (!(ok = mbar_wait(&sh.t_empty[tb], ((j >> 1) & 1) ^ 1))) break;
        const uint32_t d = tmem + tb * 128;
#pragma unroll 1
        for (int h = 0; h < 2 && ok; ++h) {   // (Gf, S^f), then (Gb, S^b)
          const int hj = 2 * j + h;
          // (the last CTA: it runs no text chain and always has frames)
          const bool stall = p.stall == VDA_TEST_STALL_OPERANDS && blockIdx.x == gridDim.x - 1 && hj == 0;
          if (!(ok = mbar_wait_or_stall(&sh.full[h], (hj >> 1) & 1, &sh.never, stall))) break;
          tc_fence_after();
          const uint32_t g = smem_u32(ring + h * kSlot), sv = g + kMat;
#pragma unroll
          for (int k = 0; k < 16; ++k) {      // G S^T (k < 8), then S G^T
            const uint32_t off = ((k % 8) / 4) * kBox + (k % 4) * 32;
            const uint64_t a = smem_desc((k < 8 ? g : sv) + off, 16, 1024, kSwizzle128B);
            const uint64_t b = smem_desc((k < 8 ? sv : g) + off, 16, 1024, kSwizzle128B);
            mma_bf16_ss(d, a, b, kIdescKK, (h | k) ? 1u : 0u);
          }
          mma_commit(&sh.empty[h]);
        }
        if (ok) mma_commit(&sh.t_full[tb]);
      }
      if (!ok) set_abort(sh, p.err);
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // epilogue: W1 = -acc from TMEM, dB = Gf + Gb from the bf16 adjoints.
    const bool leader = (warp == 2 && lane == 0);
    uint8_t* w1s = stg;
    uint8_t* dbs = stg + kMat;
    for (int j = 0; j < J; ++j) {
      const int tb = j & 1;
      const int f = f_begin + j;
      // dB's operands, the row of Gf and of Gb (bf16, just brought into L2 by
      // the producer's loads), loaded before the wait so that their latency
      // overlaps the frame's MMAs.
      uint4 ga[16], gb[16];
      {
        const __nv_bfloat16* gf = p.Gf + ((size_t)f * 128 + row) * 128;
        const __nv_bfloat16* gbp = p.Gb + ((size_t)f * 128 + row) * 128;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          ga[c] = *reinterpret_cast<const uint4*>(gf + 8 * c);
          gb[c] = *reinterpret_cast<const uint4*>(gbp + 8 * c);
        }
      }
      bool ok = !aborted(sh) && mbar_wait(&sh.t_full[tb], (j >> 1) & 1);
      if (!ok) set_abort(sh, p.err);
      if (named_bar_or(kEpiBar, 128, !ok)) break;   // one decision for the four warps
      tc_fence_after();
      if (leader) bulk_wait_read<0>();       // the previous frame's stores have read the staging
      named_bar_sync(kEpiBar, 128);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem + tb * 128 + lane_off + q * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) v[e] = -__uint_as_float(r[8 * jj + e]);
          *reinterpret_cast<uint4*>(w1s + kimg(row, q * 4 + jj)) = pack8(v);
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.t_empty[tb]);
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&ga[c]);
        const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&gb[c]);
        float v[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x = __bfloat1622float2(a2[e]), y = __bfloat1622float2(b2[e]);
          v[2 * e] = x.x + y.x;
          v[2 * e + 1] = x.y + y.y;
        }
        *reinterpret_cast<uint4*>(dbs + kimg(row, c)) = pack8(v);
      }
      fence_proxy_async_smem();
      named_bar_sync(kEpiBar, 128);
      if (leader) {
        tma_store_3d(&p.mW, w1s, 0, 0, f);
        tma_store_3d(&p.mW, w1s + kBox, 64, 0, f);
        tma_store_3d(&p.mW, dbs, 0, 128, f);
        tma_store_3d(&p.mW, dbs + kBox, 64, 128, f);
        bulk_commit();
      }
    }
    if (leader) bulk_wait<0>();               // the stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_bwd_operands_tc(const vda_problem& p, const __nv_bfloat16* Gf, const __nv_bfloat16* Gb,
                                   const __nv_bfloat16* SF, const __nv_bfloat16* SB, const float* M, const float* Bm,
                                   __nv_bfloat16* W, __nv_bfloat16* Wt, unsigned* err, cudaStream_t st) {
  BwdOperandsParams prm;
  memset(&prm, 0, sizeof(prm));
  const int heads = p.B * p.H, frames = heads * p.T;
  if (!make_bf16_rows_map(&prm.mGf, Gf, 128, frames, 128) || !make_bf16_rows_map(&prm.mSf, SF, 128, frames, 128) ||
      !make_bf16_rows_map(&prm.mGb, Gb, 128, frames, 128) || !make_bf16_rows_map(&prm.mSb, SB, 128, frames, 128) ||
      !make_bf16_rows_map(&prm.mW, W, 256, frames, 128))
    return cudaErrorInvalidValue;
  prm.Gf = Gf;
  prm.Gb = Gb;
  prm.M = reinterpret_cast<const uint8_t*>(M);
  prm.Bm = Bm;
  prm.Wt = p.n_txt > 0 ? Wt : nullptr;
  prm.err = err;
  prm.frames = frames;
  prm.heads = heads;
  prm.T = p.T;
  prm.inv_lam = 1.f / p.lambda;
  prm.stall = p.test_stall;
  const size_t smem = 1024 + kStage + 2 * kMat + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(bwd_operands_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = frames < sms ? frames : sms;
  // A text chain costs about as much as 8 frames; the weight is capped so
  // that every CTA's share of (frames + weight * heads) covers its text:
  // (frames + w heads) / grid >= w, i.e. w <= frames / (grid - heads).
  prm.text_weight = 0;
  if (prm.Wt && grid > heads) prm.text_weight = min(8, frames / (grid - heads));
  // Programmatic dependent launch: the CTAs start as the adjoint scan's CTAs
  // finish; griddep_wait() holds them until the adjoints are written.
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
  return cudaLaunchKernelEx(&cfg, bwd_operands_tc_kernel, prm);
}

}  // namespace vda
