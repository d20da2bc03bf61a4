// Single-token state update over a slot-indexed state pool (decode).
//
// "ufo.work" page §4.1 and its second article §4.1: a persistent pool of per-request states
// and a light kernel doing h_new = exp(Delta A) h_old + Delta B x for one token.  The
// kernel is bound by HBM traffic on the pool (read + write of R x dim x dstate float32),
// so the per-channel work is done once: a thread owns G consecutive states of one
// (request, channel) -- a whole channel when dstate <= 16 -- loads them with 16-byte vectors
// and keeps them in registers; Delta = softplus(delta + bias), the gate and the D term are
// evaluated once per channel.  B and C of the request are staged in shared memory once per
// block (every channel of the request reads the same values).  Consecutive threads take
// consecutive channels, so a warp streams one contiguous run of the pool row.  When a
// channel is split over several threads (dstate > 16) their partial C.h go through shared
// memory.  dstate = 16 has a kernel of its own that streams the pool through shared memory
// (state_update16_bulk_kernel, below).  With ZOH the input coefficient is the zero-order
// hold's (a - 1)/A instead of Delta (zoh_coef2 in common.cuh).
#pragma once

#include "common.cuh"

namespace ssm {

struct UpdateArgs {
  float *pool;
  const int32_t *slot_ids;
  const void *u, *delta, *z, *B, *C;
  const float *A, *Dskip, *bias;
  void *y;
  int64_t num_slots, R, dim;
  int64_t x_stride, bc_stride;  // row strides of [R][dim] and [R][dstate] inputs
  int dstate;
  int tpc;  // threads per channel = dstate / G
};

constexpr int kUpdateThreads = 256;
constexpr int kUpdateMaxState = 256;

// Grid: x over the channels of one request (kUpdateThreads / tpc per block), y strides over
// the requests.  G states per thread (4, 8 or 16; G divides dstate).
template <typename T, typename TO, bool HAS_Z, int G, bool ZOH>
__global__ void __launch_bounds__(kUpdateThreads) state_update_kernel(const UpdateArgs args) {
  constexpr bool kFast = Elem<T>::kFast;
  static_assert(G % 4 == 0 && G <= 16, "state group");
  __shared__ __align__(16) float Bs[kUpdateMaxState], Cs[kUpdateMaxState];
  __shared__ float red[kUpdateThreads];
  const int N = args.dstate, tpc = args.tpc;
  const int cpb = kUpdateThreads / tpc;  // channels per block
  const int cl = threadIdx.x / tpc, part = threadIdx.x % tpc;
  const int64_t d = int64_t(blockIdx.x) * cpb + cl;
  const bool valid = cl < cpb && d < args.dim;
  const int s0 = part * G;  // first state of this thread
  for (int64_t r = blockIdx.y; r < args.R; r += gridDim.y) {
    const int64_t slot = args.slot_ids[r];
    if (slot < 0 || slot >= args.num_slots) {  // uniform over the block: the row is skipped
      if (blockIdx.x == 0 && threadIdx.x == 0) report_status(4 /* SSM_ERR_BAD_SLOT */);
      continue;
    }
    __syncthreads();  // the previous request's B, C and partial sums are consumed
    for (int i = threadIdx.x; i < N; i += kUpdateThreads) {
      Bs[i] = Elem<T>::to_f32(static_cast<const T *>(args.B)[r * args.bc_stride + i]);
      Cs[i] = Elem<T>::to_f32(static_cast<const T *>(args.C)[r * args.bc_stride + i]);
    }
    __syncthreads();
    float acc = 0.f, uval = 0.f;
    if (valid) {
      const int64_t xo = r * args.x_stride + d;
      uval = Elem<T>::to_f32(static_cast<const T *>(args.u)[xo]);
      const float dt = softplus_t<kFast>(Elem<T>::to_f32(static_cast<const T *>(args.delta)[xo]) +
                                         (args.bias ? args.bias[d] : 0.f));
      const float2 dtl = make_float2(dt * kLog2e, dt * kLog2e);
      const float2 dtu = make_float2(dt * uval, dt * uval);
      float4 *hp = reinterpret_cast<float4 *>(args.pool + (slot * args.dim + d) * N + s0);
      const float4 *ap = reinterpret_cast<const float4 *>(args.A + d * N + s0);
      float4 h[G / 4], av[G / 4];
#pragma unroll
      for (int k = 0; k < G / 4; ++k) {
        h[k] = hp[k];
        av[k] = ap[k];
      }
      float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int k = 0; k < G / 4; ++k) {
        const float4 b4 = *reinterpret_cast<const float4 *>(Bs + s0 + 4 * k);
        const float4 c4 = *reinterpret_cast<const float4 *>(Cs + s0 + 4 * k);
        const float2 x01 = __fmul2_rn(dtl, make_float2(av[k].x, av[k].y));
        const float2 x23 = __fmul2_rn(dtl, make_float2(av[k].z, av[k].w));
        const float2 a01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
        const float2 a23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
        float2 q01 = dtu, q23 = dtu;  // input coefficient times u
        if constexpr (ZOH) {
          const float2 DT = make_float2(dt, dt), U = make_float2(uval, uval), L = make_float2(kLn2, kLn2);
          const float2 i01 = make_float2(inv_or_zero(av[k].x), inv_or_zero(av[k].y));
          const float2 i23 = make_float2(inv_or_zero(av[k].z), inv_or_zero(av[k].w));
          q01 = __fmul2_rn(U, zoh_coef2(DT, __fmul2_rn(x01, L), a01, i01));
          q23 = __fmul2_rn(U, zoh_coef2(DT, __fmul2_rn(x23, L), a23, i23));
        }
        const float2 h01 = __ffma2_rn(a01, make_float2(h[k].x, h[k].y), __fmul2_rn(q01, make_float2(b4.x, b4.y)));
        const float2 h23 = __ffma2_rn(a23, make_float2(h[k].z, h[k].w), __fmul2_rn(q23, make_float2(b4.z, b4.w)));
        acc2 = __ffma2_rn(make_float2(c4.x, c4.y), h01, acc2);
        acc2 = __ffma2_rn(make_float2(c4.z, c4.w), h23, acc2);
        h[k] = make_float4(h01.x, h01.y, h23.x, h23.y);
      }
#pragma unroll
      for (int k = 0; k < G / 4; ++k) hp[k] = h[k];
      acc = acc2.x + acc2.y;
    }
    if (tpc > 1) {  // the channel's partial sums, in thread order
      red[threadIdx.x] = acc;
      __syncthreads();
      if (valid && part == 0)
        for (int p = 1; p < tpc; ++p) acc += red[threadIdx.x + p];
    }
    if (valid && part == 0) {
      float v = fmaf(args.Dskip ? args.Dskip[d] : 0.f, uval, acc);
      if constexpr (HAS_Z) v *= silu_t<kFast>(Elem<T>::to_f32(static_cast<const T *>(args.z)[r * args.x_stride + d]));
      static_cast<TO *>(args.y)[r * args.x_stride + d] = Elem<TO>::from_f32(v);
    }
  }
}

// dstate = 16 with the pool streamed through shared memory.  A block owns one group of
// kUpdBulkCh channels and walks the requests r = blockIdx.y, blockIdx.y + gridDim.y, ...; the
// group's slice of a pool row (kUpdBulkCh x 16 float32, contiguous) comes in by one bulk copy
// issued kUpdBulkStages requests ahead of its use, and the updated slice goes back by one bulk
// store, so several slices per block are in flight while the threads compute.  A, Dskip and the
// bias of the group stay in registers across requests.  Lane l = 4j + m of warp w holds state
// quad m of channels 32w + 8k + j (k = 0..3), so each shared-memory access of a warp covers 512
// contiguous bytes; Delta, Delta u and the gate are evaluated once per channel (by lane
// 4j + m for channel 32w + 8m + j) and passed by shuffles, and C.h is reduced over the 4 lanes
// of a channel.  Waits are bounded: on a timeout the block stops (SSM_ERR_TIMEOUT),
// after a bounded wait for the copies it has in flight, and stores nothing more.
constexpr int kUpdBulkCh = 256;
constexpr int kUpdBulkStages = 3;
constexpr uint32_t kUpdBulkSlice = uint32_t(kUpdBulkCh) * 16u * 4u;
constexpr size_t kUpdBulkSmem = size_t(kUpdBulkStages) * kUpdBulkSlice;

template <typename T, typename TO, bool HAS_Z, bool ZOH>
__global__ void __launch_bounds__(kUpdateThreads, 4) state_update16_bulk_kernel(const UpdateArgs args) {
  constexpr bool kFast = Elem<T>::kFast;
  constexpr int N = 16, S = kUpdBulkStages;
  static_assert(kUpdateThreads == kUpdBulkCh, "one warp per 32 channels of the group");
  extern __shared__ __align__(128) unsigned char upd_smem[];
  float4 *const slices = reinterpret_cast<float4 *>(upd_smem);  // [S][kUpdBulkCh][4]
  __shared__ __align__(8) uint64_t full[S];
  __shared__ int64_t slot_sh[S];

  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int j = lane >> 2, m = lane & 3;
  const int64_t c0 = int64_t(blockIdx.x) * kUpdBulkCh;  // first channel of the group
  const int nch = int(min64(kUpdBulkCh, args.dim - c0));
  const uint32_t bytes = uint32_t(nch) * uint32_t(N * sizeof(float));
  const int64_t rb = blockIdx.y, nrb = gridDim.y;
  const int64_t nmine = rb < args.R ? (args.R - rb + nrb - 1) / nrb : 0;  // requests of this block
  const int cw = 32 * warp;                                                // warp's first channel
  const int own = cw + 8 * m + j;                                          // this lane's channel
  const bool own_ok = own < nch;

  float4 av[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int c = cw + 8 * k + j;
    av[k] = c < nch ? *reinterpret_cast<const float4 *>(args.A + (c0 + c) * N + 4 * m) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float Dd = (own_ok && args.Dskip) ? args.Dskip[c0 + own] : 0.f;
  const float bias = (own_ok && args.bias) ? args.bias[c0 + own] : 0.f;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    mbar_init_fence();
  }
  __syncthreads();

  // thread 0: bring request i's slice into stage i % S (a bad slot id completes the stage's
  // phase without a copy and marks it skipped)
  auto issue = [&](int64_t i) {
    const int s = int(i % S);
    const int64_t r = rb + i * nrb;
    const int64_t slot = args.slot_ids[r];
    if (slot < 0 || slot >= args.num_slots) {
      if (blockIdx.x == 0) report_status(4 /* SSM_ERR_BAD_SLOT */);
      slot_sh[s] = -1;
      mbar_arrive(&full[s]);
    } else {
      slot_sh[s] = slot;
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(slices + size_t(s) * kUpdBulkCh * 4, args.pool + (slot * args.dim + c0) * N, bytes, &full[s]);
    }
  };
  if (threadIdx.x == 0)
    for (int64_t i = 0; i < min64(S, nmine); ++i) issue(i);

  for (int64_t i = 0; i < nmine; ++i) {
    const int s = int(i % S);
    const int64_t r = rb + i * nrb;
    // the request's token inputs, read while its slice is in flight
    const T *Br = static_cast<const T *>(args.B) + r * args.bc_stride + 4 * m;
    const T *Cr = static_cast<const T *>(args.C) + r * args.bc_stride + 4 * m;
    const float4 b4 = make_float4(Elem<T>::to_f32(Br[0]), Elem<T>::to_f32(Br[1]), Elem<T>::to_f32(Br[2]),
                                  Elem<T>::to_f32(Br[3]));
    const float4 c4 = make_float4(Elem<T>::to_f32(Cr[0]), Elem<T>::to_f32(Cr[1]), Elem<T>::to_f32(Cr[2]),
                                  Elem<T>::to_f32(Cr[3]));
    float dtl = 0.f, dtu = 0.f, uval = 0.f, zval = 0.f;
    const int64_t xo = r * args.x_stride + c0 + own;
    if (own_ok) {
      uval = Elem<T>::to_f32(static_cast<const T *>(args.u)[xo]);
      const float dt = softplus_t<kFast>(Elem<T>::to_f32(static_cast<const T *>(args.delta)[xo]) + bias);
      dtl = dt * kLog2e;
      dtu = ZOH ? uval : dt * uval;
      if constexpr (HAS_Z) zval = Elem<T>::to_f32(static_cast<const T *>(args.z)[xo]);
    }
    const bool landed = mbar_wait_bounded(&full[s], uint32_t((i / S) & 1));
    const int64_t slot = slot_sh[s];
    float4 *sl = slices + size_t(s) * kUpdBulkCh * 4;
    float own_sum = 0.f;
    if (slot >= 0 && landed) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // channel cw + 8k + j belongs to lane 4j + k
        const float l2 = __shfl_sync(0xffffffffu, dtl, 4 * j + k);
        const float du = __shfl_sync(0xffffffffu, dtu, 4 * j + k);
        const int c = cw + 8 * k + j;
        const float4 h = sl[c * 4 + m];  // past the group's end: stale, never stored
        const float2 L2 = make_float2(l2, l2), DU = make_float2(du, du);
        const float2 x01 = __fmul2_rn(L2, make_float2(av[k].x, av[k].y));
        const float2 x23 = __fmul2_rn(L2, make_float2(av[k].z, av[k].w));
        const float2 a01 = make_float2(ex2_approx(x01.x), ex2_approx(x01.y));
        const float2 a23 = make_float2(ex2_approx(x23.x), ex2_approx(x23.y));
        float2 q01 = DU, q23 = DU;  // input coefficient times u
        if constexpr (ZOH) {
          const float2 L = make_float2(kLn2, kLn2), DT = __fmul2_rn(L2, L);
          const float2 i01 = make_float2(inv_or_zero(av[k].x), inv_or_zero(av[k].y));
          const float2 i23 = make_float2(inv_or_zero(av[k].z), inv_or_zero(av[k].w));
          q01 = __fmul2_rn(DU, zoh_coef2(DT, __fmul2_rn(x01, L), a01, i01));
          q23 = __fmul2_rn(DU, zoh_coef2(DT, __fmul2_rn(x23, L), a23, i23));
        }
        const float2 h01 = __ffma2_rn(a01, make_float2(h.x, h.y), __fmul2_rn(q01, make_float2(b4.x, b4.y)));
        const float2 h23 = __ffma2_rn(a23, make_float2(h.z, h.w), __fmul2_rn(q23, make_float2(b4.z, b4.w)));
        sl[c * 4 + m] = make_float4(h01.x, h01.y, h23.x, h23.y);
        float2 p2 = __fmul2_rn(make_float2(c4.x, c4.y), h01);
        p2 = __ffma2_rn(make_float2(c4.z, c4.w), h23, p2);
        float part = p2.x + p2.y;
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if (k == m) own_sum = part;  // channel cw + 8m + j is this lane's own
      }
    }
    fence_proxy_async_smem();  // the updated slice is read by the bulk store below
    if (__syncthreads_or(!landed)) {
      // a copy did not land within the bounded wait (SSM_ERR_TIMEOUT is recorded): stop, once
      // more waiting (bounded) for the copies still in flight so that none writes shared
      // memory after the block has exited
      if (threadIdx.x == 0) {
        for (int64_t q = i; q < min64(i + S, nmine); ++q) mbar_wait_bounded(&full[q % S], uint32_t((q / S) & 1));
        bulk_wait_all();
      }
      return;
    }
    if (slot >= 0 && own_ok) {
      float v = fmaf(Dd, uval, own_sum);
      if constexpr (HAS_Z) v *= silu_t<kFast>(zval);
      static_cast<TO *>(args.y)[xo] = Elem<TO>::from_f32(v);
    }
    if (threadIdx.x == 0) {
      if (slot >= 0) {
        bulk_s2g(args.pool + (slot * args.dim + c0) * N, sl, bytes);
        bulk_commit();
        bulk_wait_read_all();  // the stage is refilled next
      }
      if (i + S < nmine) issue(i + S);
    }
  }
  if (threadIdx.x == 0) bulk_wait_all();
}

}  // namespace ssm
