// Backward pass of the selective scan (gradients for training), in time segments.
//
// Schedule ("ufo.work" page, §2.2, strategy B: keep checkpoints, recompute the rest; its
// second article, §3.1: chunk-boundary states and the composition of chunk operators).  The
// sequence is cut into segments of seg_len steps so that every (sequence, segment, channel
// tile) is a unit of its own and even one long sequence fills the GPU:
//
//  1. bwd_seg_kernel, per unit, in forward order from a zero state: the zero-start state hz
//     entering every 8-step block (the block's checkpoint) and the sum of Delta from the
//     segment start to the block (exp(A sum) is the block's decay from the segment start); at
//     the segment end hz (the segment's forward operator applied to zero), the sum of Delta
//     over the segment (its decay exp(A sum)) and the zero-start adjoint
//         G = sum_t (prod_{k <= t} a_k) C_t dyraw_t,
//     which the segment passes to the step before it when no adjoint enters from its end (with
//     mu entering from the end it passes exp(A sum) mu + G).
//  2. bwd_seg_scan_kernel, per (sequence, channel, state): the segment operators composed
//     forwards from h0 (the true state entering each segment) and backwards from dh_last (the
//     true adjoint entering each segment from its end).
//  3. seq_bwd_kernel, per unit: walks the segment from its end.  For every 8-step block it
//     recomputes a_t = exp(Delta_t A) and h_t from the block's state hz + exp(A sum) h_start,
//     keeping them in registers, and runs the adjoint recurrence backwards through the block:
//
//   dyraw_t  = dy_t silu(z_t)                 dz_t = dy_t yraw_t silu'(z_t)
//   dh      += dyraw_t C_t                    (y_t reads h_t)
//   dC_t    += dyraw_t h_t                    dB_t += dh Delta_t u_t       (summed over channels)
//   du_t     = dyraw_t D + Delta_t sum_n dh B_t
//   dDelta_t = sum_n (dh h_{t-1} a_t A + dh B_t u_t)      ddelta_t = dDelta_t sigmoid(delta_t + bias)
//   dA      += dh h_{t-1} a_t Delta_t         dh *= a_t                   (on to h_{t-1})
//
// with yraw_t = sum_n C_t h_t + D u_t (the ungated output).  With the zero-order hold the input
// coefficient Delta becomes c = (a - 1) / A per state (zoh_coef2): dB_t += dh c u, du_t =
// dyraw D + sum_n dh c B, dDelta_t = sum_n dh a (h_{t-1} A + B u) (dc/dDelta = a), and dA gains
// dh B u dc/dA (zoh_dcdA2).  dh starts from the adjoint that
// enters the segment from its end and, in the first segment, ends as dh0.  Each forward
// exponential is evaluated twice (segment pass, recompute), none a third time.
//
// Lanes: LPC = 4 lanes share a channel and split its states (NS = N / 4 each); a warp holds
// 8 channels, a CTA W warps.  Per block a lane evaluates the per-step terms (softplus, its
// derivative, the gate) for 2 of the 8 steps and hands them to the channel's other lanes by
// shuffles; sums over the states (yraw, du, dDelta) are reduced across those 4 lanes.  The
// sums over channels (dB, dC) go through a per-warp buffer in shared memory: every lane writes
// its per-state terms of four steps at a time, then lane (which, n) of the warp adds the warp's
// 8 channels for those four steps and adds them to dB or dC with one 16-byte vector atomic in
// global memory (scalar atomics where the rows do not allow it).  dA, dDskip and dbias are
// summed in registers and added with atomics once per unit.
//
// Staging is the forward's: TMA bulk copies of the u, delta, z, dy rows and the B, C rows of a
// chunk, double-buffered, with B and C widened to float32 in a [step][state] layout once per
// chunk.  Segments are whole chunks.
#pragma once

#include "common.cuh"
#include "seq_scan.cuh"

namespace ssm {

struct BwdArgs {
  const void *dy;          // [batch][dim][seqlen], dtype TG, strides as u
  const float *dh_last;    // [batch][dim][N] or nullptr
  void *du, *ddelta, *dz;  // [batch][dim][seqlen], dtype TG
  float *dA, *dDskip, *dbias, *dh0;
  float *dB, *dC;          // [batch][N][seqlen], zero on entry to the walk (summed by atomics)
  float *ckpt;             // [batch][nblk][dim][N]: zero-start state of the segment entering each block
  float *cumd;             // [batch][nblk][dim]: sum of Delta from the segment start to the block
  float *seg_sum;          // [batch][nseg][dim]: sum of Delta over the segment
  float *seg_h;            // [batch][nseg][dim][N]: zero-start final state; after the scan: state entering
  float *seg_g;            // [batch][nseg][dim][N]: zero-start adjoint; after the scan: adjoint from the end
  int64_t nblk;            // blocks per sequence: ceil(seqlen / 8)
  int64_t seg_len;         // steps per segment (a multiple of the chunk)
  int nseg;                // segments per sequence
  int vec_dbc;             // dB, dC rows take 16-byte vector atomics
};

// sigmoid(x) from w = e^-|x| (which the softplus already has): 1/(1+w) for x > 0, w/(1+w) else.
__device__ __forceinline__ float sigmoid_from_w(float x, float w) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + w));
  return (x > 0.f ? 1.f : w) * r;
}

// softplus(x) from one exponential (the forward kernels' softplus_fast) and, when asked for,
// sigmoid(x), its derivative, from the same exponential
template <bool kFast, bool kSig> __device__ __forceinline__ float softplus_sig(float x, float &sgm) {
  if constexpr (kFast) {
    const float w = ex2_approx(-fabsf(x) * kLog2e);
    float q = fmaf(w, -0.00853909645229578f, 0.044089239090681076f);
    q = fmaf(w, q, -0.10768117010593414f);
    q = fmaf(w, q, 0.17745204269886017f);
    q = fmaf(w, q, -0.24495449662208557f);
    q = fmaf(w, q, 0.33275479078292847f);
    q = fmaf(w, q, -0.4999740421772003f);
    q = fmaf(w, q, 0.9999998211860657f);
    if constexpr (kSig) sgm = sigmoid_from_w(x, w);
    return fmaf(w, q, fmaxf(x, 0.f));
  } else {
    if constexpr (kSig) sgm = 1.f / (1.f + expf(-x));
    return softplus_precise(x);
  }
}

// Zero-order hold: the derivative of the input coefficient c = (e^x - 1) / A (x = Delta A) with
// respect to A, dc/dA = (Delta a - c) / A = Delta^2 psi(x), psi(x) = (x e^x - e^x + 1) / x^2.
// Where |x| < 1/4 the difference cancels, so the series psi = sum_{k>=2} (k-1)/k! x^(k-2) =
// 1/2 + x/3 + x^2/8 + x^3/30 + x^4/144 + x^5/840 is taken (truncation below |x|^6/5760 <
// 1e-7 relative); elsewhere the direct form loses at most a few ulp to the cancellation.  As in
// zoh_coef2 both branches are evaluated and selected (the unselected one may be inf/nan).
// (The derivative with respect to Delta is dc/dDelta = a.)
__device__ __forceinline__ float2 zoh_dcdA2(float2 dt, float2 x, float2 a, float2 c, float2 invA) {
  float2 s = __ffma2_rn(x, make_float2(1.f / 840.f, 1.f / 840.f), make_float2(1.f / 144.f, 1.f / 144.f));
  s = __ffma2_rn(x, s, make_float2(1.f / 30.f, 1.f / 30.f));
  s = __ffma2_rn(x, s, make_float2(0.125f, 0.125f));
  s = __ffma2_rn(x, s, make_float2(1.f / 3.f, 1.f / 3.f));
  s = __ffma2_rn(x, s, make_float2(0.5f, 0.5f));
  const float2 near = __fmul2_rn(__fmul2_rn(dt, dt), s);
  const float2 far = __fmul2_rn(__ffma2_rn(dt, a, make_float2(-c.x, -c.y)), invA);
  return make_float2(fabsf(x.x) < 0.25f ? near.x : far.x, fabsf(x.y) < 0.25f ? near.y : far.y);
}

template <typename T, typename TG, int N, int TC, int W>
struct BwdCfg {
  static constexpr int kN = N;
  static constexpr int kTC = TC;
  static constexpr int kLPC = 4;
  static constexpr int kNS = N / kLPC;
  static constexpr int kCPW = 32 / kLPC;  // 8 channels per warp
  static constexpr int kWarps = W;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kCT = kWarps * kCPW;
  static constexpr int kSub = 8 / kLPC;   // steps of an 8-step block a lane prepares: 2
  static constexpr int kXP = TC + 8;      // staged row pitch (elements), as in the forward
  static constexpr size_t kXElems = size_t(3) * kCT * kXP;     // u, delta, z
  static constexpr size_t kYElems = size_t(kCT) * kXP;         // dy (dtype TG)
  static constexpr size_t kBCElems = size_t(2) * N * TC;
  static constexpr int kCOff = TC * N + 16;
  static constexpr size_t kBFElems = size_t(2) * TC * N + 16;
  // per warp: the per-state dB, dC terms of half an 8-step block, [2 step pairs][CPW channels]
  // [2 N states][2 steps] (the two halves of a block leave the buffer one after the other); in a
  // channel's row dB's terms come first for even channels and dC's first for odd ones, and odd
  // channels swap the two 16-byte halves of every 32-byte group, so that both the lanes' 16-byte
  // writes and the per-(which, n) float2 column reads are free of bank conflicts
  static constexpr size_t kPartElems = size_t(2) * kCPW * 2 * N * 2;
  static constexpr size_t kOffY = 2 * kXElems * sizeof(T);
  static constexpr size_t kOffBC = kOffY + 2 * kYElems * sizeof(TG);
  static constexpr size_t kOffBF = (kOffBC + 2 * kBCElems * sizeof(T) + 15) / 16 * 16;
  static constexpr size_t kOffPart = kOffBF + 2 * kBFElems * sizeof(float);
  static constexpr size_t kSmemBytes = kOffPart + kWarps * kPartElems * sizeof(float);
  static constexpr size_t kSegSmemBytes = kOffPart;  // the segment pass needs the staging only
  static_assert(kNS % 4 == 0, "whole float4 groups of states per lane");
  static_assert(2 * N == 32 && kNS == 4, "one (which, state) pair per lane in the dB/dC reduction");
  static_assert(TC % 8 == 0 && (kXP * sizeof(T)) % 16 == 0 && (kXP * sizeof(TG)) % 16 == 0, "16-byte rows");
  static_assert(kOffY % 16 == 0 && kOffBF % 16 == 0 && kOffPart % 16 == 0, "aligned buffers");
};

// Where a unit's work lies: unit = (sequence s, segment, channel tile), tiles fastest.
struct BwdUnit {
  int tile, seg, s;
  int64_t d0, t_lo, t_hi;
  int c_lo, c_hi;  // chunks [c_lo, c_hi)
};
template <int TC, int CT>
__device__ __forceinline__ BwdUnit bwd_unit(const ScanArgs &args, const BwdArgs &bw, int unit) {
  BwdUnit w;
  w.tile = unit % args.ntiles;
  const int rest = unit / args.ntiles;
  w.seg = rest % bw.nseg;
  w.s = rest / bw.nseg;
  w.d0 = int64_t(w.tile) * CT;
  w.t_lo = int64_t(w.seg) * bw.seg_len;
  w.t_hi = min64(args.seqlen, w.t_lo + bw.seg_len);
  w.c_lo = int(w.t_lo / TC);
  w.c_hi = int((w.t_hi + TC - 1) / TC);
  return w;
}

// TMA staging of chunk cc: the u, delta (and z) rows and the dy rows of the tile and the B, C
// rows of the chunk window, into buffer `buf`, completing on `bar`.
template <typename Cfg, typename T, typename TG>
__device__ __forceinline__ void bwd_stage(const ScanArgs &args, const BwdArgs &bw, T *xs0, TG *ys0, T *bcs0,
                                          uint64_t *bar, int buf, int cc, int nx, int nvalid, int64_t d0,
                                          int64_t xbase, int64_t bcbase) {
  constexpr int CT = Cfg::kCT, NT = Cfg::kThreads, XP = Cfg::kXP, N = Cfg::kN, TC = Cfg::kTC;
  constexpr int V = Elem<T>::kVec;
  const int64_t seqlen_r = (args.seqlen + V - 1) / V * V;
  const int64_t wstart = int64_t(cc) * TC;
  const int64_t wend = min64(wstart + TC, seqlen_r);
  const uint32_t rows_t = uint32_t((wend - wstart) * int64_t(sizeof(T)));
  const uint32_t rows_g = uint32_t((wend - wstart) * int64_t(sizeof(TG)));
  T *xd = xs0 + buf * Cfg::kXElems;
  TG *yd = ys0 + buf * Cfg::kYElems;
  T *bd = bcs0 + buf * Cfg::kBCElems;
  fence_proxy_async_smem();
  if (threadIdx.x == 0)
    mbar_arrive_expect_tx(bar, rows_t * uint32_t(nx * nvalid + 2 * N) + rows_g * uint32_t(nvalid));
  for (int r = threadIdx.x; r < (nx + 1) * CT + 2 * N; r += NT) {
    if (r < nx * CT) {
      const int which = r / CT, c2 = r % CT;
      if (c2 >= nvalid) continue;
      const T *base = static_cast<const T *>(which == 0 ? args.u : (which == 1 ? args.delta : args.z));
      bulk_g2s(xd + size_t(r) * XP, base + xbase + (d0 + c2) * args.x_dim_stride + wstart, rows_t, bar);
    } else if (r < (nx + 1) * CT) {
      const int c2 = r - nx * CT;
      if (c2 >= nvalid) continue;
      bulk_g2s(yd + size_t(c2) * XP, static_cast<const TG *>(bw.dy) + xbase + (d0 + c2) * args.x_dim_stride + wstart,
               rows_g, bar);
    } else {
      const int r2 = r - (nx + 1) * CT, which = r2 / N, n = r2 % N;
      const T *base = static_cast<const T *>(which == 0 ? args.B : args.C);
      bulk_g2s(bd + size_t(r2) * TC, base + bcbase + int64_t(n) * args.bc_state_stride + wstart, rows_t, bar);
    }
  }
}

// B and C of a staged chunk widened to float32, [step][state] (C at kCOff)
template <typename Cfg, typename T>
__device__ __forceinline__ void bwd_widen(const T *bs, float *bfw) {
  constexpr int N = Cfg::kN, TC = Cfg::kTC;
  for (int i = threadIdx.x; i < 2 * N * (TC / 8); i += Cfg::kThreads) {
    const int row = i % (2 * N), blk = i / (2 * N);
    float f[8];
    load_sub<T, 8>(bs + size_t(row) * TC + blk * 8, f);
    float *dst = bfw + (row >= N ? Cfg::kCOff : 0) + blk * 8 * N + row % N;
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j * N] = f[j];
  }
}

// ---------------------------------------------------------------------------------------------
// 1. The segment pass.
#ifndef SSM_BWD_SEG_WARPS_PER_SM
#define SSM_BWD_SEG_WARPS_PER_SM 20  // resident warps per SM the segment pass is compiled for (96 registers)
#endif
template <typename T, typename TG, int N, int TC, int W, bool HAS_Z, bool ZOH>
__global__ void __launch_bounds__(W * 32, SSM_BWD_SEG_WARPS_PER_SM / W) bwd_seg_kernel(const ScanArgs args, const BwdArgs bw) {
  using Cfg = BwdCfg<T, TG, N, TC, W>;
  constexpr int LPC = Cfg::kLPC, NS = Cfg::kNS, CPW = Cfg::kCPW, CT = Cfg::kCT;
  constexpr int XP = Cfg::kXP, SUB = Cfg::kSub;
  constexpr bool kFast = Elem<T>::kFast;
  constexpr int nx = HAS_Z ? 3 : 2;

  extern __shared__ __align__(16) unsigned char smem[];
  T *const xs0 = reinterpret_cast<T *>(smem);
  TG *const ys0 = reinterpret_cast<TG *>(smem + Cfg::kOffY);
  T *const bcs0 = reinterpret_cast<T *>(smem + Cfg::kOffBC);
  float *const bf0 = reinterpret_cast<float *>(smem + Cfg::kOffBF);
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int unit_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane % LPC, c = lane / LPC;
  const int ch = warp * CPW + c;
  const int lbase = lane - g;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init_fence();
  }
  __syncthreads();
  uint32_t gc = 0;

  for (;;) {
    if (threadIdx.x == 0) unit_sh = int(atomicAdd(args.ticket, 1u));
    __syncthreads();
    const int unit = unit_sh;
    if (unit >= args.total_units) break;
    const BwdUnit w = bwd_unit<TC, CT>(args, bw, unit);
    const int nvalid = int(min64(CT, args.dim - w.d0));
    const int64_t d = w.d0 + ch;
    const bool ch_ok = d < args.dim;
    const int64_t xbase = int64_t(w.s) * args.x_batch_stride;
    const int64_t bcbase = int64_t(w.s) * args.bc_batch_stride;

    float2 A2[NS / 2], hz[NS / 2], pp[NS / 2], gb[NS / 2];
    [[maybe_unused]] float2 IA[NS / 2];  // 1/A (zero-order hold)
    float bias = 0.f, cd = 0.f;
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
      A2[p] = hz[p] = gb[p] = make_float2(0.f, 0.f);
      pp[p] = make_float2(1.f, 1.f);
      if constexpr (ZOH) IA[p] = make_float2(0.f, 0.f);
    }
    if (ch_ok) {
      const float *Ar = args.A + d * N + g * NS;
#pragma unroll
      for (int p = 0; p < NS / 2; ++p) {
        A2[p] = make_float2(Ar[2 * p] * kLog2e, Ar[2 * p + 1] * kLog2e);
        if constexpr (ZOH) IA[p] = make_float2(inv_or_zero(Ar[2 * p]), inv_or_zero(Ar[2 * p + 1]));
      }
      bias = args.bias ? args.bias[d] : 0.f;
    }

    // one 8-step block, first step first
    auto block = [&](auto masked_tag, const T *X, const TG *Y, const float *Bf, int64_t wstart, int sb) {
      constexpr bool kMasked = decltype(masked_tag)::value;
      const int k0 = sb * 8;
      const int64_t gblk = (wstart + k0) / 8;
      const int rel_hi = int(min64(w.t_hi - (wstart + k0), 8));
      const int c0 = k0 + g * SUB;
      float uv[SUB], dv[SUB], gv[SUB], dm[SUB], um[SUB], rm[SUB];
      [[maybe_unused]] float zv[SUB];
      load_sub<T, SUB>(X + size_t(ch) * XP + c0, uv);
      load_sub<T, SUB>(X + size_t(CT + ch) * XP + c0, dv);
      if constexpr (HAS_Z) load_sub<T, SUB>(X + size_t(2 * CT + ch) * XP + c0, zv);
      load_sub<TG, SUB>(Y + size_t(ch) * XP + c0, gv);
#pragma unroll
      for (int j = 0; j < SUB; ++j) {
        float unused;
        const float dt = softplus_sig<kFast, false>(dv[j] + bias, unused);
        float dyr = gv[j];
        if constexpr (HAS_Z) dyr *= silu_t<kFast>(zv[j]);
        const bool in = ch_ok && (!kMasked || g * SUB + j < rel_hi);  // stale rows stay out
        dm[j] = in ? dt : 0.f;
        um[j] = in ? (ZOH ? uv[j] : dt * uv[j]) : 0.f;  // the input's factor besides B: Delta u, or u
        rm[j] = in ? dyr : 0.f;
      }
      float dl[8], dU[8], dr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        dl[k] = __shfl_sync(0xffffffffu, dm[k % SUB], lbase + k / SUB);
        dU[k] = __shfl_sync(0xffffffffu, um[k % SUB], lbase + k / SUB);
        dr[k] = __shfl_sync(0xffffffffu, rm[k % SUB], lbase + k / SUB);
      }
      if (ch_ok) {
        const int64_t bo = (int64_t(w.s) * bw.nblk + gblk) * args.dim + d;
        float *ck = bw.ckpt + bo * N + g * NS;
#pragma unroll
        for (int q = 0; q < NS / 4; ++q)
          reinterpret_cast<float4 *>(ck)[q] = make_float4(hz[2 * q].x, hz[2 * q].y, hz[2 * q + 1].x, hz[2 * q + 1].y);
        if (g == 0) bw.cumd[bo] = cd;
      }
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int t = k0 + k;
        const float2 dd = make_float2(dl[k], dl[k]), uu = make_float2(dU[k], dU[k]), rr = make_float2(dr[k], dr[k]);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
          float4 b4 = reinterpret_cast<const float4 *>(Bf + t * N + g * NS)[q];
          float4 c4 = reinterpret_cast<const float4 *>(Bf + Cfg::kCOff + t * N + g * NS)[q];
          if constexpr (kMasked) {
            if (k >= rel_hi) b4 = c4 = make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = 2 * q + e;
            const float2 bp = e ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y);
            const float2 cp = e ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
            const float2 x = __fmul2_rn(dd, A2[p]);
            const float2 a = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            float2 q = uu;
            if constexpr (ZOH) q = __fmul2_rn(uu, zoh_coef2(dd, __fmul2_rn(x, make_float2(kLn2, kLn2)), a, IA[p]));
            hz[p] = __ffma2_rn(a, hz[p], __fmul2_rn(q, bp));
            pp[p] = __fmul2_rn(pp[p], a);
            gb[p] = __ffma2_rn(pp[p], __fmul2_rn(rr, cp), gb[p]);
          }
        }
        cd += dl[k];
      }
    };

    if (w.c_hi > w.c_lo)
      bwd_stage<Cfg>(args, bw, xs0, ys0, bcs0, &bars[gc & 1u], int(gc & 1u), w.c_lo, nx, nvalid, w.d0, xbase, bcbase);
    for (int cc = w.c_lo; cc < w.c_hi; ++cc, ++gc) {
      const int buf = int(gc & 1u);
      const int64_t wstart = int64_t(cc) * TC;
      const bool landed = mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);
      bwd_widen<Cfg>(bcs0 + buf * Cfg::kBCElems, bf0 + buf * Cfg::kBFElems);
      // chunk cc widened; every warp is done with chunk cc-1's buffers
      if (__syncthreads_or(!landed)) {
        mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);  // no copy left writing shared memory
        return;
      }
      if (cc + 1 < w.c_hi)
        bwd_stage<Cfg>(args, bw, xs0, ys0, bcs0, &bars[buf ^ 1], buf ^ 1, cc + 1, nx, nvalid, w.d0, xbase, bcbase);
      const T *X = xs0 + buf * Cfg::kXElems;
      const TG *Y = ys0 + buf * Cfg::kYElems;
      const float *Bf = bf0 + buf * Cfg::kBFElems;
#pragma unroll 1
      for (int sb = 0; sb < TC / 8; ++sb) {
        if (wstart + sb * 8 >= w.t_hi) break;  // uniform
        if (wstart + sb * 8 + 8 <= w.t_hi)
          block(std::false_type{}, X, Y, Bf, wstart, sb);
        else
          block(std::true_type{}, X, Y, Bf, wstart, sb);
      }
    }
    if (ch_ok) {
      const int64_t o = (int64_t(w.s) * bw.nseg + w.seg) * args.dim + d;
#pragma unroll
      for (int q = 0; q < NS / 4; ++q) {
        reinterpret_cast<float4 *>(bw.seg_h + o * N + g * NS)[q] =
            make_float4(hz[2 * q].x, hz[2 * q].y, hz[2 * q + 1].x, hz[2 * q + 1].y);
        reinterpret_cast<float4 *>(bw.seg_g + o * N + g * NS)[q] =
            make_float4(gb[2 * q].x, gb[2 * q].y, gb[2 * q + 1].x, gb[2 * q + 1].y);
      }
      if (g == 0) bw.seg_sum[o] = cd;
    }
    __syncthreads();  // shared state of this unit is dead before the next unit overwrites it
  }
}

// ---------------------------------------------------------------------------------------------
// 2. The segment scan: one thread per (sequence, channel, state).  Forwards, seg_h becomes the
// state entering each segment (from h0); backwards, seg_g becomes the adjoint entering each
// segment from its end (from dh_last).
__global__ void __launch_bounds__(256) bwd_seg_scan_kernel(const float *A, const float *h0, const float *dh_last,
                                                           const float *seg_sum, float *seg_h, float *seg_g,
                                                           int64_t batch, int64_t dim, int N, int nseg) {
  const int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= batch * dim * N) return;
  const int64_t dn = e % (dim * N), s = e / (dim * N);
  const int64_t d = dn / N, n = dn % N;
  const float A2 = A[dn] * kLog2e;
  // Segments in batches of 8: a batch's loads are all issued before its results are written
  // back in place, so they are in flight together (the values do not depend on h or mu).
  constexpr int Q = 8;
  float P[Q], gz[Q];
  float h = h0 ? h0[e] : 0.f;
  for (int q0 = 0; q0 < nseg; q0 += Q) {
#pragma unroll
    for (int i = 0; i < Q; ++i) {
      const int q = q0 + i;
      if (q < nseg) {
        const int64_t o = (s * nseg + q) * dim + d;
        P[i] = seg_sum[o];
        gz[i] = seg_h[o * N + n];
      }
    }
#pragma unroll
    for (int i = 0; i < Q; ++i) {
      const int q = q0 + i;
      if (q < nseg) {
        const int64_t o = (s * nseg + q) * dim + d;
        seg_h[o * N + n] = h;
        h = fmaf(ex2_approx(A2 * P[i]), h, gz[i]);
      }
    }
  }
  float mu = dh_last ? dh_last[e] : 0.f;
  for (int q0 = nseg - 1; q0 >= 0; q0 -= Q) {
#pragma unroll
    for (int i = 0; i < Q; ++i) {
      const int q = q0 - i;
      if (q >= 0) {
        const int64_t o = (s * nseg + q) * dim + d;
        P[i] = seg_sum[o];
        gz[i] = seg_g[o * N + n];
      }
    }
#pragma unroll
    for (int i = 0; i < Q; ++i) {
      const int q = q0 - i;
      if (q >= 0) {
        const int64_t o = (s * nseg + q) * dim + d;
        seg_g[o * N + n] = mu;
        mu = fmaf(ex2_approx(A2 * P[i]), mu, gz[i]);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// 3. The walk.
#ifndef SSM_BWD_WARPS_PER_SM
#define SSM_BWD_WARPS_PER_SM 12  // resident warps per SM the walk is compiled for (its register budget)
#endif
#ifndef SSM_BWD_ZOH_WARPS_PER_SM
#define SSM_BWD_ZOH_WARPS_PER_SM 8  // the same for the zero-order-hold walk (no spills at 8)
#endif
template <typename T, typename TG, int N, int TC, int W, bool HAS_Z, bool ZOH>
__global__ void __launch_bounds__(W * 32, (ZOH ? SSM_BWD_ZOH_WARPS_PER_SM : SSM_BWD_WARPS_PER_SM) / W)
    seq_bwd_kernel(const ScanArgs args, const BwdArgs bw) {
  using Cfg = BwdCfg<T, TG, N, TC, W>;
  constexpr int LPC = Cfg::kLPC, NS = Cfg::kNS, CPW = Cfg::kCPW, CT = Cfg::kCT, NT = Cfg::kThreads;
  constexpr int XP = Cfg::kXP, SUB = Cfg::kSub;
  constexpr bool kFast = Elem<T>::kFast;
  constexpr int nx = HAS_Z ? 3 : 2;

  extern __shared__ __align__(16) unsigned char smem[];
  T *const xs0 = reinterpret_cast<T *>(smem);                                   // [2][3][CT][XP]
  TG *const ys0 = reinterpret_cast<TG *>(smem + Cfg::kOffY);                    // [2][CT][XP]
  T *const bcs0 = reinterpret_cast<T *>(smem + Cfg::kOffBC);                    // [2][2][N][TC]
  float *const bf0 = reinterpret_cast<float *>(smem + Cfg::kOffBF);             // [2][kBFElems]
  float *const part0 = reinterpret_cast<float *>(smem + Cfg::kOffPart);         // [W][kPartElems]
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int unit_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane % LPC, c = lane / LPC;
  const int ch = warp * CPW + c;
  const int lbase = lane - g;
  const int64_t L = args.seqlen;
  float *const part = part0 + size_t(warp) * Cfg::kPartElems;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init_fence();
  }
  __syncthreads();
  uint32_t gc = 0;

  for (;;) {
    if (threadIdx.x == 0) unit_sh = int(atomicAdd(args.ticket, 1u));
    __syncthreads();
    const int unit = unit_sh;
    if (unit >= args.total_units) break;
    const BwdUnit w = bwd_unit<TC, CT>(args, bw, unit);
    const int s = w.s;
    const int64_t d0 = w.d0;
    const int nvalid = int(min64(CT, args.dim - d0));
    const int64_t d = d0 + ch;
    const bool ch_ok = d < args.dim;
    const int64_t xbase = int64_t(s) * args.x_batch_stride;
    const int64_t bcbase = int64_t(s) * args.bc_batch_stride;
    const int64_t so = (int64_t(s) * bw.nseg + w.seg) * args.dim + d;  // this segment's row
    // The checkpoint (zero-start state entering a block) and the sum of Delta from the segment
    // start to the block, for the block the walk takes next: blocks are taken last first, one
    // after the other, and each block's values are loaded while the block before it is walked.
    float4 ckn[NS / 4];
    float cdn = 0.f;
#pragma unroll
    for (int q = 0; q < NS / 4; ++q) ckn[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    const int64_t blk_lo = w.t_lo / 8;  // the segment's first block (segments are whole chunks)
    auto load_ckpt = [&](int64_t gb) {
      if (ch_ok && gb >= blk_lo) {
        const int64_t bo = (int64_t(s) * bw.nblk + gb) * args.dim + d;
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) ckn[q] = reinterpret_cast<const float4 *>(bw.ckpt + bo * N + g * NS)[q];
        cdn = bw.cumd[bo];
      }
    };
    if (w.t_hi > w.t_lo) load_ckpt((w.t_hi - 1) / 8);  // the segment's last block comes first

    float2 A2[NS / 2], An[NS / 2], dh[NS / 2], dAacc[NS / 2], hs[NS / 2];
    [[maybe_unused]] float2 IA[NS / 2];  // 1/A (zero-order hold)
    float bias = 0.f, Dd = 0.f, dDacc = 0.f, dbacc = 0.f;
#pragma unroll
    for (int p = 0; p < NS / 2; ++p) {
      A2[p] = An[p] = dh[p] = dAacc[p] = hs[p] = make_float2(0.f, 0.f);
      if constexpr (ZOH) IA[p] = make_float2(0.f, 0.f);
    }
    if (ch_ok) {
      const float *Ar = args.A + d * N + g * NS;
      const float *mr = bw.seg_g + so * N + g * NS;  // the adjoint entering from the segment's end
      const float *hr = bw.seg_h + so * N + g * NS;  // the state entering the segment
#pragma unroll
      for (int p = 0; p < NS / 2; ++p) {
        An[p] = make_float2(Ar[2 * p], Ar[2 * p + 1]);
        A2[p] = make_float2(An[p].x * kLog2e, An[p].y * kLog2e);
        if constexpr (ZOH) IA[p] = make_float2(inv_or_zero(An[p].x), inv_or_zero(An[p].y));
        dh[p] = make_float2(mr[2 * p], mr[2 * p + 1]);
        hs[p] = make_float2(hr[2 * p], hr[2 * p + 1]);
      }
      bias = args.bias ? args.bias[d] : 0.f;
      Dd = args.Dskip ? args.Dskip[d] : 0.f;
    }

    // dB, dC terms of four steps (chunk-local steps t0 .. t0 + 3, buffer slots 0..3): lane
    // (which, n) adds up the warp's 8 channels for the four steps and adds them to dB or dC
    auto reduce_part = [&](int64_t wstart, int t0) {
      __syncwarp();
      const int which = lane / N, n = lane % N;
      float v[4];
#pragma unroll
      for (int kp = 0; kp < 2; ++kp) {  // steps t0 + 2 kp and t0 + 2 kp + 1
        float2 sum = make_float2(0.f, 0.f);
#pragma unroll
        for (int cc = 0; cc < CPW; ++cc) {
          const int word = ((((which ^ (cc & 1)) * N) + n) * 2) ^ ((cc & 1) << 2);
          sum = __fadd2_rn(sum, *reinterpret_cast<const float2 *>(part + (size_t(kp) * CPW + cc) * (4 * N) + word));
        }
        v[2 * kp] = sum.x;
        v[2 * kp + 1] = sum.y;
      }
      __syncwarp();  // the terms are consumed before the buffer is rewritten
      const int64_t gt = wstart + t0;
      if (gt < L) {
        float *dst = (which ? bw.dC : bw.dB) + (int64_t(s) * N + n) * L + gt;
        if (bw.vec_dbc) {
          atomicAdd(reinterpret_cast<float4 *>(dst), make_float4(v[0], v[1], v[2], v[3]));  // L % 4 == 0
        } else {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            if (gt + kk < L) atomicAdd(dst + kk, v[kk]);
        }
      }
    };

    // one 8-step block, from the end of the block to its start
    auto block = [&](auto masked_tag, const T *X, const TG *Y, const float *Bf, int64_t wstart, int sb) {
      constexpr bool kMasked = decltype(masked_tag)::value;
      const int k0 = sb * 8;                      // chunk-local first step of the block
      const int64_t gblk = (wstart + k0) / 8;     // block index in the sequence
      const int rel_hi = int(min64(L - (wstart + k0), 8));  // steps of the block inside the sequence
      // ---- this lane's SUB steps: softplus, its derivative, the gate
      const int c0 = k0 + g * SUB;
      float uv[SUB], dv[SUB], gv[SUB], dm[SUB], um[SUB], sg[SUB];
      [[maybe_unused]] float zv[SUB], zs[SUB], zd[SUB];
      load_sub<T, SUB>(X + size_t(ch) * XP + c0, uv);
      load_sub<T, SUB>(X + size_t(CT + ch) * XP + c0, dv);
      if constexpr (HAS_Z) load_sub<T, SUB>(X + size_t(2 * CT + ch) * XP + c0, zv);
      load_sub<TG, SUB>(Y + size_t(ch) * XP + c0, gv);
#pragma unroll
      for (int j = 0; j < SUB; ++j) {
        float sgm;
        float dt = softplus_sig<kFast, true>(dv[j] + bias, sgm);
        float du = ZOH ? uv[j] : dt * uv[j], gy = gv[j];  // the input's factor besides B: Delta u, or u
        // a channel past the end of a ragged tile, or a step past the end of the sequence, takes
        // no part (its staged rows are stale; selects keep non-finite values out of the sums)
        const bool in = ch_ok && (!kMasked || g * SUB + j < rel_hi);
        dt = in ? dt : 0.f;
        du = in ? du : 0.f;
        gy = in ? gy : 0.f;
        dm[j] = dt;
        um[j] = du;
        sg[j] = sgm;
        gv[j] = gy;
        if constexpr (HAS_Z) {
          // silu(z) = z s, silu'(z) = s (1 + z (1 - s)), s = sigmoid(z)
          const float s_ = kFast ? fmaf(0.5f, tanh_approx(0.5f * zv[j]), 0.5f) : 1.f / (1.f + expf(-zv[j]));
          zs[j] = zv[j] * s_;
          zd[j] = s_ * fmaf(zv[j], 1.f - s_, 1.f);
        }
      }
      float dl[8], dU[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        dl[k] = __shfl_sync(0xffffffffu, dm[k % SUB], lbase + k / SUB);
        dU[k] = __shfl_sync(0xffffffffu, um[k % SUB], lbase + k / SUB);
      }
      // ---- recompute a_t and h_t over the block from its state: the segment's zero-start
      // state plus the state entering the segment, decayed to the block
      float2 hin[NS / 2];
#pragma unroll
      for (int p = 0; p < NS / 2; ++p) hin[p] = make_float2(0.f, 0.f);
      float4 ckv[NS / 4];
#pragma unroll
      for (int q = 0; q < NS / 4; ++q) ckv[q] = ckn[q];
      const float cdv = cdn;
      load_ckpt(gblk - 1);  // in flight while this block is walked
      if (ch_ok) {
        const float2 cd2 = make_float2(cdv, cdv);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
          const float4 v = ckv[q];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = 2 * q + e;
            const float2 x = __fmul2_rn(cd2, A2[p]);
            const float2 dec = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            hin[p] = __ffma2_rn(dec, hs[p], e ? make_float2(v.z, v.w) : make_float2(v.x, v.y));
          }
        }
      }
      float2 a[8][NS / 2], h[8][NS / 2];
      float yp[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int t = k0 + k;
        const float2 dd = make_float2(dl[k], dl[k]), uu = make_float2(dU[k], dU[k]);
        float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
          float4 b4 = reinterpret_cast<const float4 *>(Bf + t * N + g * NS)[q];
          float4 c4 = reinterpret_cast<const float4 *>(Bf + Cfg::kCOff + t * N + g * NS)[q];
          if constexpr (kMasked) {
            if (k >= rel_hi) b4 = c4 = make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = 2 * q + e;
            const float2 bp = e ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y);
            const float2 cp = e ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
            const float2 x = __fmul2_rn(dd, A2[p]);
            a[k][p] = make_float2(ex2_approx(x.x), ex2_approx(x.y));
            float2 q = uu;
            if constexpr (ZOH) q = __fmul2_rn(uu, zoh_coef2(dd, __fmul2_rn(x, make_float2(kLn2, kLn2)), a[k][p], IA[p]));
            h[k][p] = __ffma2_rn(a[k][p], k ? h[k - 1][p] : hin[p], __fmul2_rn(q, bp));
            acc2 = __ffma2_rn(cp, h[k][p], acc2);
          }
        }
        yp[k] = acc2.x + acc2.y;
      }
      // ---- sum C h over the channel's lanes for this lane's steps (recursive halving)
#pragma unroll
      for (int lev = 0; (1 << lev) < LPC; ++lev) {
        const int off = LPC >> (lev + 1), half = 8 >> (lev + 1);
        const bool upper = (g & off) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
          const float send = upper ? yp[j] : yp[half + j];
          const float keep = upper ? yp[half + j] : yp[j];
          yp[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      // ---- the gate's gradient and the ungated output's, for this lane's steps
      float dym[SUB], dzv[SUB];
#pragma unroll
      for (int j = 0; j < SUB; ++j) {
        const float yraw = fmaf(Dd, uv[j], yp[j]);
        if constexpr (HAS_Z) {
          dzv[j] = gv[j] * yraw * zd[j];
          dym[j] = gv[j] * zs[j];
        } else {
          dzv[j] = 0.f;
          dym[j] = gv[j];
        }
        {
          const bool in = ch_ok && (!kMasked || g * SUB + j < rel_hi);  // zero, whatever z and u hold
          dzv[j] = in ? dzv[j] : 0.f;
          dym[j] = in ? dym[j] : 0.f;
          uv[j] = in ? uv[j] : 0.f;
        }
      }
      float dr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) dr[k] = __shfl_sync(0xffffffffu, dym[k % SUB], lbase + k / SUB);
      // ---- the adjoint recurrence, last step first.  S1 = sum_n dh c B (c = Delta for Euler:
      // the factor Delta is applied after the sum), S2 = sum_n dh h_{t-1} a A, and for the
      // zero-order hold S3 = sum_n dh a B (dc/dDelta = a)
      float s1[8], s2[8];
      [[maybe_unused]] float s3[8];
      float2 hb[2], hc[2];  // dB, dC terms of the odd step, written with the even step below it
#pragma unroll
      for (int k = 7; k >= 0; --k) {
        const int t = k0 + k;
        const float2 dd = make_float2(dl[k], dl[k]), uu = make_float2(dU[k], dU[k]);
        const float2 dyr = make_float2(dr[k], dr[k]);
        float2 S1 = make_float2(0.f, 0.f), S2 = make_float2(0.f, 0.f);
        [[maybe_unused]] float2 S3 = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < NS / 4; ++q) {
          float4 b4 = reinterpret_cast<const float4 *>(Bf + t * N + g * NS)[q];
          float4 c4 = reinterpret_cast<const float4 *>(Bf + Cfg::kCOff + t * N + g * NS)[q];
          if constexpr (kMasked) {
            if (k >= rel_hi) b4 = c4 = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          float2 tb[2], tc[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int p = 2 * q + e;
            const float2 bp = e ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y);
            const float2 cp = e ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
            dh[p] = __ffma2_rn(dyr, cp, dh[p]);                 // y_t reads h_t
            tc[e] = __fmul2_rn(dyr, h[k][p]);                    // dC_t term of this channel
            const float2 daa = __fmul2_rn(__fmul2_rn(dh[p], k ? h[k - 1][p] : hin[p]), a[k][p]);
            S2 = __ffma2_rn(daa, An[p], S2);                     // sum_n dh h_{t-1} a A
            dAacc[p] = __ffma2_rn(daa, dd, dAacc[p]);            // dA += dh h_{t-1} a Delta
            if constexpr (ZOH) {
              const float2 x = __fmul2_rn(__fmul2_rn(dd, A2[p]), make_float2(kLn2, kLn2));
              const float2 cz = zoh_coef2(dd, x, a[k][p], IA[p]);
              tb[e] = __fmul2_rn(dh[p], __fmul2_rn(cz, uu));     // dB_t term: dh c u
              const float2 db = __fmul2_rn(dh[p], bp);
              S1 = __ffma2_rn(db, cz, S1);                       // sum_n dh c B
              S3 = __ffma2_rn(db, a[k][p], S3);                  // sum_n dh a B
              // dA += dh B u dc/dA
              dAacc[p] = __ffma2_rn(__fmul2_rn(db, uu), zoh_dcdA2(dd, x, a[k][p], cz, IA[p]), dAacc[p]);
            } else {
              tb[e] = __fmul2_rn(dh[p], uu);                     // dB_t term: dh Delta u
              S1 = __ffma2_rn(dh[p], bp, S1);                    // sum_n dh B
            }
            dh[p] = __fmul2_rn(dh[p], a[k][p]);                  // on to h_{t-1}
          }
          if (k & 1) {
            hb[0] = tb[0];
            hb[1] = tb[1];
            hc[0] = tc[0];
            hc[1] = tc[1];
          } else {
            // steps k and k + 1 of the lane's four states as (step k, step k + 1) pairs
            float *prow = part + (size_t((k & 3) >> 1) * CPW + c) * (4 * N);
            const int sw = (c & 1) * 4;
            float *pb = prow + ((c & 1) * N + g * NS) * 2;        // dB terms
            float *pc = prow + ((1 - (c & 1)) * N + g * NS) * 2;  // dC terms
            *reinterpret_cast<float4 *>(pb + sw) = make_float4(tb[0].x, hb[0].x, tb[0].y, hb[0].y);
            *reinterpret_cast<float4 *>(pb + 4 - sw) = make_float4(tb[1].x, hb[1].x, tb[1].y, hb[1].y);
            *reinterpret_cast<float4 *>(pc + sw) = make_float4(tc[0].x, hc[0].x, tc[0].y, hc[0].y);
            *reinterpret_cast<float4 *>(pc + 4 - sw) = make_float4(tc[1].x, hc[1].x, tc[1].y, hc[1].y);
          }
        }
        s1[k] = S1.x + S1.y;
        s2[k] = S2.x + S2.y;
        if constexpr (ZOH) s3[k] = S3.x + S3.y;
        if (k == 4) reduce_part(wstart, k0 + 4);  // steps 4..7 done: their terms leave the buffer
      }
      reduce_part(wstart, k0);
      // ---- sums over the channel's lanes of sum_n dh B and sum_n dh h a A, for this lane's steps
#pragma unroll
      for (int lev = 0; (1 << lev) < LPC; ++lev) {
        const int off = LPC >> (lev + 1), half = 8 >> (lev + 1);
        const bool upper = (g & off) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
          const float send1 = upper ? s1[j] : s1[half + j], keep1 = upper ? s1[half + j] : s1[j];
          const float send2 = upper ? s2[j] : s2[half + j], keep2 = upper ? s2[half + j] : s2[j];
          s1[j] = keep1 + __shfl_xor_sync(0xffffffffu, send1, off);
          s2[j] = keep2 + __shfl_xor_sync(0xffffffffu, send2, off);
          if constexpr (ZOH) {
            const float send3 = upper ? s3[j] : s3[half + j], keep3 = upper ? s3[half + j] : s3[j];
            s3[j] = keep3 + __shfl_xor_sync(0xffffffffu, send3, off);
          }
        }
      }
      if (ch_ok) {
        float odu[SUB], odd[SUB];
#pragma unroll
        for (int j = 0; j < SUB; ++j) {
          if constexpr (ZOH) {
            odu[j] = fmaf(dym[j], Dd, s1[j]);                    // du = dyraw D + sum dh c B
            odd[j] = fmaf(uv[j], s3[j], s2[j]) * sg[j];          // (sum dh h a A + u sum dh a B) sigmoid
          } else {
            odu[j] = fmaf(dym[j], Dd, dm[j] * s1[j]);            // du = dyraw D + Delta sum dh B
            odd[j] = fmaf(uv[j], s1[j], s2[j]) * sg[j];          // (sum dh h a A + u sum dh B) sigmoid
          }
          if constexpr (kMasked) {
            const bool in = g * SUB + j < rel_hi;
            odd[j] = in ? odd[j] : 0.f;
            odu[j] = in ? odu[j] : 0.f;
          }
          dDacc = fmaf(dym[j], uv[j], dDacc);
          dbacc += odd[j];
        }
        const int64_t off = xbase + d * args.x_dim_stride + wstart + c0;
        TG *gdu = static_cast<TG *>(bw.du) + off;
        TG *gdd = static_cast<TG *>(bw.ddelta) + off;
        [[maybe_unused]] TG *gdz = HAS_Z ? static_cast<TG *>(bw.dz) + off : nullptr;
        if (!kMasked || g * SUB + SUB <= rel_hi) {
          store_sub<TG, SUB>(gdu, odu);
          store_sub<TG, SUB>(gdd, odd);
          if constexpr (HAS_Z) store_sub<TG, SUB>(gdz, dzv);
        } else {
#pragma unroll
          for (int j = 0; j < SUB; ++j)
            if (g * SUB + j < rel_hi) {
              gdu[j] = Elem<TG>::from_f32(odu[j]);
              gdd[j] = Elem<TG>::from_f32(odd[j]);
              if constexpr (HAS_Z) gdz[j] = Elem<TG>::from_f32(dzv[j]);
            }
        }
      }
    };

    // ------------------------------------------------------------- the segment's chunks, last first
    if (w.c_hi > w.c_lo)
      bwd_stage<Cfg>(args, bw, xs0, ys0, bcs0, &bars[gc & 1u], int(gc & 1u), w.c_hi - 1, nx, nvalid, d0, xbase,
                     bcbase);
    for (int cc = w.c_hi - 1; cc >= w.c_lo; --cc, ++gc) {
      const int buf = int(gc & 1u);
      const int64_t wstart = int64_t(cc) * TC;
      const bool landed = mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);
      bwd_widen<Cfg>(bcs0 + buf * Cfg::kBCElems, bf0 + buf * Cfg::kBFElems);
      // chunk cc widened; every warp is done with chunk cc+1's buffers
      if (__syncthreads_or(!landed)) {
        mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);  // no copy left writing shared memory
        return;
      }
      if (cc > w.c_lo)
        bwd_stage<Cfg>(args, bw, xs0, ys0, bcs0, &bars[buf ^ 1], buf ^ 1, cc - 1, nx, nvalid, d0, xbase, bcbase);
      const T *X = xs0 + buf * Cfg::kXElems;
      const TG *Y = ys0 + buf * Cfg::kYElems;
      const float *Bf = bf0 + buf * Cfg::kBFElems;
#pragma unroll 1
      for (int sb = TC / 8 - 1; sb >= 0; --sb) {
        if (wstart + sb * 8 >= L) continue;  // a block wholly past the end (uniform)
        if (wstart + sb * 8 + 8 <= L)
          block(std::false_type{}, X, Y, Bf, wstart, sb);
        else
          block(std::true_type{}, X, Y, Bf, wstart, sb);
      }
    }

    // ------------------------------------------------------------- per-unit results
    if (ch_ok) {
      if (bw.dh0 && w.seg == 0) {
        float *hr = bw.dh0 + (int64_t(s) * args.dim + d) * N + g * NS;
#pragma unroll
        for (int p = 0; p < NS / 2; ++p) {
          hr[2 * p] = dh[p].x;
          hr[2 * p + 1] = dh[p].y;
        }
      }
#pragma unroll
      for (int p = 0; p < NS / 2; ++p) {
        atomicAdd(bw.dA + d * N + g * NS + 2 * p, dAacc[p].x);
        atomicAdd(bw.dA + d * N + g * NS + 2 * p + 1, dAacc[p].y);
      }
    }
    // dDskip and dbias: this lane's steps, summed over the channel's lanes
#pragma unroll
    for (int off = 1; off < LPC; off *= 2) {
      dDacc += __shfl_xor_sync(0xffffffffu, dDacc, off);
      dbacc += __shfl_xor_sync(0xffffffffu, dbacc, off);
    }
    if (ch_ok && g == 0) {
      if (bw.dDskip) atomicAdd(bw.dDskip + d, dDacc);
      if (bw.dbias) atomicAdd(bw.dbias + d, dbacc);
    }
    __syncthreads();  // shared state of this unit is dead before the next unit overwrites it
  }
}

}  // namespace ssm
