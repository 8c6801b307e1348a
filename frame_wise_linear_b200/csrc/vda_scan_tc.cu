// Bidirectional scan on tcgen05 tensor cores (bf16 path, d_k = d_v = 128).
//
// "VDN-H3" (comfyui-wiki.com), section on how Video DeltaNet speeds up H3: a
// bidirectional linear branch carries context through a constant-size state;
// "VDN-MiniMax-H3" (aiezz.com), section 03: the text is written once into
// both directional states.  Per (b, h) and direction, every step is
//     X = S_prev + B_t / lambda,    S_t = M_t X          (M_t = lambda A_t^{-1})
// starting from S_prev = 0 on the text slot (which gives S_0), then frames
// 1..T (forward) or T..1 (backward).  S^f_t / S^b_t are written as float32.
//
// Precision: M_t arrives as bf16 hi + lo (written by the factor step in the
// MMA operand layout); X is split the same way; the product is
// M_hi X_hi + M_hi X_lo + M_lo X_hi in float32 (the dropped M_lo X_lo term is
// below 2^-16 relative).  X_hi and X_lo sit side by side as one operand of
// 2N columns, so M_hi [X_hi | X_lo] is one N = 2N pass, and M_lo X_hi
// accumulates onto its first N columns; the row warps add the two halves.
// (The step is bound by shared-memory bandwidth: the TMA writes of M_t and
// B_t, X, the state staging and the MMAs' operand reads; this form reads
// M_hi once instead of twice.)  ||M_t||_2 <= 1, so the
// per-step error does not grow along the chain.  Each state goes out as
// bfloat16 in the readout's operand layout (row-major, d_k x d_v); float32
// states are written as well when the caller asks for them.
//
// The recurrence is independent per column of S, so each chain is split over
// kSplit CTAs of N = 128 / kSplit columns.  CTA layout (288 threads):
//   warps 0..7  own TMEM lanes = rows of S (two warps per lane quarter, 32
//               columns each): build X (row m) in shared memory from S_{t-1}
//               and B_t, stage the previous state (swizzled) for a TMA store
//               while the step's MMAs run, then read S_t back from TMEM;
//   warp 8      one thread: bulk-copies M_t (64 KB) into a 2-stage ring and
//               B_t (this CTA's columns) by TMA as soon as the row warps have
//               copied the previous one into registers, and issues the 16
//               MMAs of each step.
// Every wait is bounded; a timeout sets the error bit and the CTA winds down.
#include "sm100.cuh"
#include "vda_internal.cuh"

namespace vda {
namespace {

using namespace sm100;

constexpr int kSplit = 2;
constexpr int N = 128 / kSplit;              // columns of S per CTA
constexpr int kRowWarps = 8;                 // two per TMEM lane quarter
constexpr int kMmaWarp = kRowWarps;
constexpr int kCols = N / 2;                 // columns of S per row thread
constexpr int kThreads = 32 * (kRowWarps + 1);
static_assert(N == 64 && kCols == 32, "row warps hold one 32-column TMEM load and one 128-byte X row");
constexpr int kMBytes = 65536;               // M_t hi | lo
constexpr int kXHalf = (N / 64) * 16384;     // X hi (or lo): N/64 blocks of 128 rows x 128 B
constexpr int kSStage = N * 128 * 4;         // S_t staging: N/32 boxes of 128 rows x 128 B
constexpr int kBBuf = N * 128 * 4;           // B_t columns of this CTA, same layout
constexpr int kEpiBar = 1;                   // named barrier of the row warps
constexpr int kAhead = 4;                    // steps of M_t and B_t prefetched into L2
constexpr uint32_t kIdesc = idesc_bf16_f32(128, N, /*a MN*/ false, /*b MN*/ true);
constexpr uint32_t kIdesc2 = idesc_bf16_f32(128, 2 * N, /*a MN*/ false, /*b MN*/ true);

struct ScanTcParams {
  CUtensorMap mSFb, mSBb;  // states for the readout: [frames][128][128] bfloat16, 64 x 128 boxes
  CUtensorMap mSF, mSB;    // optional float32 states: [frames * 128][128], 32 x 128 boxes
  CUtensorMap mB;          // [slots * 128][128] float32, 32 x 128 boxes
  const uint8_t* M;        // per slot 64 KB: M hi (32 KB) | M lo (32 KB)
  const float* Bm;         // per slot 128 x 128 float
  unsigned* err;
  int T;
  int f32_out;             // also write the float32 states
  int b_frames;            // B is [frames * 128][128] with no text rows; the text step adds nothing
  float lam;
  int stall;               // testing hook: a VDA_TEST_STALL_* site, 0 in normal use
};

struct Shared {
  uint64_t m_full[2], m_empty[2];
  uint64_t x_full, d_full, b_full, b_empty;
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

__global__ void __launch_bounds__(kThreads, 1) scan_tc_kernel(const __grid_constant__ ScanTcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* mring = base;                     // 2 x 64 KB
  uint8_t* xbuf = base + 2 * kMBytes;        // X hi | X lo
  uint8_t* sstage = xbuf + 2 * kXHalf;       // S_t staging
  uint8_t* bbuf = sstage + kSStage;          // B_t (this CTA's columns)
  Shared& sh = *reinterpret_cast<Shared*>(bbuf + kBBuf);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int c0 = blockIdx.x * N;             // first column of S handled here
  const int dir = blockIdx.y;
  const int bh = blockIdx.z;
  const int T = p.T;
  const size_t slot0 = (size_t)bh * (T + 1);
  const bool first_cta = blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
  auto slot_of = [&](int s) -> size_t { return slot0 + (s == 0 ? 0 : (dir == 0 ? s : T + 1 - s)); };
  // First row of B_s: its slot's, or, for frame-indexed B, its frame's (the
  // text step reads frame 1's rows and the row warps ignore them).
  auto brow_of = [&](int s) -> size_t {
    if (!p.b_frames) return slot_of(s) * 128;
    const int t = s == 0 ? 1 : (dir == 0 ? s : T + 1 - s);
    return ((size_t)bh * T + (t - 1)) * 128;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.m_full[i], 1);
      mbar_init(&sh.m_empty[i], 1);
    }
    mbar_init(&sh.x_full, 32 * kRowWarps);
    mbar_init(&sh.d_full, 1);
    mbar_init(&sh.b_full, 1);
    mbar_init(&sh.b_empty, 32 * kRowWarps);
    mbar_init(&sh.drain, 1);
    mbar_init(&sh.never, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sh.tmem_base, 2 * N);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  griddep_launch_dependents();   // the readout's CTAs may take SMs as this grid's finish

  if (warp == kMmaWarp) {
    if (lane == 0) {
      // ---------------------------------------------------- loads + MMAs
      // B_s: one box per 32 columns, into the buffer the row warps build X from.
      const uint64_t pol = policy_evict_first();
      int b_last = -1;                         // last step whose B_s load was issued
      auto issue_b = [&](int s) {
        b_last = s;
        mbar_expect_tx(&sh.b_full, kBBuf);
#pragma unroll
        for (int b = 0; b < N / 32; ++b)
          tma_load_2d(bbuf + b * 16384, &p.mB, &sh.b_full, c0 + 32 * b, (int)brow_of(s), pol);
      };
      auto issue_load = [&](int s) {
        const int st = s & 1;
        const uint8_t* src = p.M + slot_of(s) * (size_t)kMBytes;
        mbar_expect_tx(&sh.m_full[st], kMBytes);
        bulk_load(mring + st * kMBytes, src, kMBytes / 2, &sh.m_full[st]);
        bulk_load(mring + st * kMBytes + kMBytes / 2, src + kMBytes / 2, kMBytes / 2, &sh.m_full[st]);
      };
      // Steps further ahead are brought into L2 by the TMA engine, so that the
      // row warps' B_t loads and the M_t copies hit L2 (one CTA of the pair).
      auto prefetch = [&](int s) {
        if (blockIdx.x != 0 || s > T) return;
        bulk_prefetch_l2(p.M + slot_of(s) * (size_t)kMBytes, kMBytes);
        bulk_prefetch_l2(p.Bm + brow_of(s) * 128, 128 * 128 * 4);
      };
      tma_prefetch_desc(&p.mB);
      griddep_wait();                // M_t and B_t come from the previous kernel
      int issued = 0;
      issue_b(0);
      issue_load(0);
      ++issued;
      if (T >= 1) {
        issue_load(1);
        ++issued;
      }
      for (int s = 1; s < kAhead; ++s) prefetch(s);
      const uint32_t maddr = smem_u32(mring);
      const uint32_t xaddr = smem_u32(xbuf);
      for (int s = 0; s <= T; ++s) {
        const int st = s & 1;
        // After a timeout the row warps run on without waiting (to keep their
        // named barrier balanced) and keep arriving on b_empty and x_full, so
        // those barriers' phases no longer say anything: stop issuing.
        if (aborted(sh)) break;
        // The row warps have copied B_s into registers: the buffer takes B_{s+1}.
        if (!mbar_wait(&sh.b_empty, s & 1)) {
          set_abort(sh, p.err);
          break;
        }
        // B_s has landed (b_full's phases move only with this thread's own
        // loads, so the wait is exact): B_{s+1}'s arrive.expect_tx can never
        // meet a phase that still waits for B_s's bytes.
        if (!mbar_wait(&sh.b_full, s & 1)) {
          set_abort(sh, p.err);
          break;
        }
        if (s + 1 <= T) issue_b(s + 1);
        const bool stall = p.stall == VDA_TEST_STALL_SCAN_OPERAND && first_cta && s == 1;
        if (!mbar_wait(&sh.m_full[st], (s >> 1) & 1) || !mbar_wait_or_stall(&sh.x_full, s & 1, &sh.never, stall)) {
          set_abort(sh, p.err);
          break;
        }
        tc_fence_after();
        prefetch(s + kAhead);
        const uint32_t ma = maddr + st * kMBytes;
        // M_hi [X_hi | X_lo] into columns 0 .. 2N-1 (X_lo is the operand's
        // second 64-column block), then M_lo X_hi onto columns 0 .. N-1.
#pragma unroll
        for (int pass = 0; pass < 2; ++pass) {
          const uint32_t a_off = pass == 1 ? kMBytes / 2 : 0;      // M lo on the second pass
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint64_t a = smem_desc(ma + a_off + (k / 4) * 16384 + (k % 4) * 32, 16, 1024, kSwizzle128B);
            const uint64_t b = smem_desc(xaddr + k * 16 * 128, kXHalf, 1024, kSwizzle128B);
            mma_bf16_ss(tmem, a, b, pass == 0 ? kIdesc2 : kIdesc, (pass | k) ? 1u : 0u);
          }
        }
        mma_commit(&sh.d_full);
        mma_commit(&sh.m_empty[st]);
        if (s + 2 <= T) {
          // refill this stage with step s + 2 once its MMAs have read it
          if (!mbar_wait(&sh.m_empty[st], (s >> 1) & 1)) {
            set_abort(sh, p.err);
            break;
          }
          issue_load(s + 2);
          ++issued;
        }
      }
      if (aborted(sh)) {  // copies still in flight land before exit
        for (int s = issued > 2 ? issued - 2 : 0; s < issued; ++s) mbar_wait(&sh.m_full[s & 1], (s >> 1) & 1);
        if (b_last >= 0) mbar_wait(&sh.b_full, b_last & 1);
      }
      mma_commit(&sh.drain);
      mbar_wait(&sh.drain, 0);
    }
  } else {
    // ---------------------------------------------------- rows of S (warps 0..7)
    const int m = (warp % 4) * 32 + lane;    // row of S = TMEM lane (warp % 4 = lane quarter)
    const int hc = warp / 4;                 // columns kCols * hc .. + kCols - 1 of this CTA's N
    const float inv_lam = 1.f / p.lam;
    float srow[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) srow[j] = 0.f;
    // S_t row m -> swizzled staging -> TMA store, while the next step's MMAs
    // run (S_{t+1} needs only srow): as bfloat16, the readout's operand (this
    // CTA's 64 columns are one 128-byte-swizzled box), and, when asked for,
    // as float32 (two 32-column boxes) through the same buffer.
    const bool leader = (warp == 0 && lane == 0);
    auto store_state = [&](int s) {
      const int t = dir == 0 ? s : T + 1 - s;
      const int frame = bh * T + (t - 1);
      if (leader) bulk_wait_read<0>();      // the previous store has read the buffer
      named_bar_sync(kEpiBar, 32 * kRowWarps);
#pragma unroll
      for (int q = 0; q < kCols / 8; ++q)
        *reinterpret_cast<uint4*>(sstage + sw128(m, (kCols / 8) * hc + q)) =
            make_uint4(pack_bf16(srow[8 * q], srow[8 * q + 1]), pack_bf16(srow[8 * q + 2], srow[8 * q + 3]),
                       pack_bf16(srow[8 * q + 4], srow[8 * q + 5]), pack_bf16(srow[8 * q + 6], srow[8 * q + 7]));
      fence_proxy_async_smem();
      named_bar_sync(kEpiBar, 32 * kRowWarps);
      if (leader) {
        tma_store_3d(dir == 0 ? &p.mSFb : &p.mSBb, sstage, c0, 0, frame);
        bulk_commit();
      }
      if (p.f32_out) {                        // the same for every thread
        if (leader) bulk_wait_read<0>();
        named_bar_sync(kEpiBar, 32 * kRowWarps);
#pragma unroll
        for (int q = 0; q < kCols / 4; ++q)
          *reinterpret_cast<float4*>(sstage + hc * 16384 + sw128(m, q)) =
              make_float4(srow[4 * q], srow[4 * q + 1], srow[4 * q + 2], srow[4 * q + 3]);
        fence_proxy_async_smem();
        named_bar_sync(kEpiBar, 32 * kRowWarps);
        if (leader) {
          const CUtensorMap* map = dir == 0 ? &p.mSF : &p.mSB;
#pragma unroll
          for (int b = 0; b < N / 32; ++b) tma_store_2d(map, sstage + b * 16384, c0 + 32 * b, frame * 128);
          bulk_commit();
        }
      }
    };
    // The loop never breaks: after a timeout the waits are skipped, so the
    // row warps always meet at the named barrier the same number of times.
    for (int s = 0; s <= T; ++s) {
      // X row m = S_{s-1} row m + B_s row m / lambda, split into hi / lo, MN-major swizzled.
      const bool okb = !aborted(sh) && mbar_wait(&sh.b_full, s & 1);
      if (!okb && !aborted(sh)) set_abort(sh, p.err);
      // B box hc (32 columns) into registers first, and the buffer back to
      // the load thread at once, so B_{s+1} is on its way while X_s is built.
      float bv[kCols];
#pragma unroll
      for (int q = 0; q < kCols / 4; ++q) {
        const float4 b4 = *reinterpret_cast<const float4*>(bbuf + hc * 16384 + sw128(m, q));
        bv[4 * q] = b4.x;
        bv[4 * q + 1] = b4.y;
        bv[4 * q + 2] = b4.z;
        bv[4 * q + 3] = b4.w;
      }
      mbar_arrive(&sh.b_empty);
      const bool no_b = p.b_frames && s == 0;   // frame-indexed B: nothing at the text step
#pragma unroll
      for (int q = 0; q < kCols / 8; ++q) {
        float h[8], l[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float x = no_b ? srow[8 * q + i] : fmaf(bv[8 * q + i], inv_lam, srow[8 * q + i]);
          h[i] = __bfloat162float(__float2bfloat16_rn(x));
          l[i] = x - h[i];
        }
        const uint32_t off = sw128(m, (kCols / 8) * hc + q);   // N = 64: one 128-byte row per k
        *reinterpret_cast<uint4*>(xbuf + off) =
            make_uint4(pack_bf16(h[0], h[1]), pack_bf16(h[2], h[3]), pack_bf16(h[4], h[5]), pack_bf16(h[6], h[7]));
        *reinterpret_cast<uint4*>(xbuf + kXHalf + off) =
            make_uint4(pack_bf16(l[0], l[1]), pack_bf16(l[2], l[3]), pack_bf16(l[4], l[5]), pack_bf16(l[6], l[7]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sh.x_full);
      if (s >= 2) store_state(s - 1);          // S_{s-1}, still in srow
      const bool stall = p.stall == VDA_TEST_STALL_SCAN_PRODUCT && first_cta && s == 1;
      const bool ok = !aborted(sh) && mbar_wait_or_stall(&sh.d_full, s & 1, &sh.never, stall);
      if (!ok && !aborted(sh)) set_abort(sh, p.err);
      tc_fence_after();
      {
        // S_t = (M_hi X_hi + M_lo X_hi) + M_hi X_lo
        uint32_t r[32], r2[32];
        const uint32_t ta = tmem + ((uint32_t)((warp % 4) * 32) << 16) + kCols * hc;
        tmem_ld_32x32b_x32(ta, r);
        tmem_ld_32x32b_x32(ta + N, r2);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < kCols; ++j) srow[j] = __uint_as_float(r[j]) + __uint_as_float(r2[j]);
      }
    }
    if (T >= 1) store_state(T);
    if (leader) bulk_wait<0>();               // S stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, 2 * N);
}

}  // namespace

cudaError_t launch_scan_tc(const vda_problem& p, const float* M, const float* Bm, __nv_bfloat16* SFb,
                           __nv_bfloat16* SBb, float* SF, float* SB, unsigned* err, cudaStream_t st,
                           bool b_frames) {
  ScanTcParams prm;
  memset(&prm, 0, sizeof(prm));
  const int frames = p.B * p.H * p.T;
  const long long brows = b_frames ? (long long)frames * 128 : (long long)p.B * p.H * (p.T + 1) * 128;
  prm.b_frames = b_frames ? 1 : 0;
  if (!make_bf16_rows_map(&prm.mSFb, SFb, 128, frames, 128) || !make_bf16_rows_map(&prm.mSBb, SBb, 128, frames, 128) ||
      !make_f32_rows_map(&prm.mB, Bm, brows, 128))
    return cudaErrorInvalidValue;
  prm.f32_out = (SF != nullptr && SB != nullptr) ? 1 : 0;
  if (prm.f32_out && (!make_f32_rows_map(&prm.mSF, SF, (long long)frames * 128, 128) ||
                      !make_f32_rows_map(&prm.mSB, SB, (long long)frames * 128, 128)))
    return cudaErrorInvalidValue;
  prm.M = reinterpret_cast<const uint8_t*>(M);
  prm.Bm = Bm;
  prm.err = err;
  prm.T = p.T;
  prm.lam = p.lambda;
  prm.stall = p.test_stall;
  const size_t smem = 1024 + 2 * kMBytes + 2 * kXHalf + kSStage + kBBuf + sizeof(Shared);
  cudaError_t e = cudaFuncSetAttribute(scan_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // Launched with programmatic stream serialization: its CTAs start as the
  // Gram+factor kernel's CTAs finish, and its load thread waits for that
  // kernel (griddep_wait) before reading M_t and B_t.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kSplit, 2, p.B * p.H);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, scan_tc_kernel, prm);
}

}  // namespace vda
