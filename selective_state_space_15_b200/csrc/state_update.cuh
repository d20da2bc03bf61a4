// Single-token state update over a slot-indexed state pool (decode).
//
// "ufo.work" page §4.1 and its second article §4.1: a persistent pool of per-request states
// and a light kernel doing h_new = exp(Delta A) h_old + Delta B x for one token.  The
// kernel is bound by HBM traffic on the pool (read + write of R x dim x dstate float32),
// so the mapping is chosen for coalescing: a thread owns 4 consecutive states (one 16-byte
// load and store) of one (request, channel); the dstate/4 threads of a channel are
// adjacent lanes and reduce C.h with shuffles; consecutive channels of a request are
// consecutive groups, so a warp streams one contiguous run of the pool row.
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
  int qlog2;  // log2(dstate / 4): lanes per channel = 1 << qlog2
};

// Grid: x covers the dim * dstate/4 items of one request (256 per block), y strides over the
// requests, so the (request, channel, quad) split needs no 64-bit division.
template <typename T, typename TO, bool HAS_Z>
__global__ void __launch_bounds__(256) state_update_kernel(const UpdateArgs args) {
  constexpr bool kFast = Elem<T>::kFast;
  const int Q = 1 << args.qlog2;
  const int N = args.dstate;
  const int item = blockIdx.x * 256 + threadIdx.x;  // < dim * Q, checked on the host
  const bool valid = item < int(args.dim) * Q;
  const int d = item >> args.qlog2, q = item & (Q - 1);
  for (int64_t r = blockIdx.y; r < args.R; r += gridDim.y) {
    const int64_t slot = args.slot_ids[r];
    if (slot < 0 || slot >= args.num_slots) {  // uniform over the block: the row is skipped
      if (blockIdx.x == 0 && threadIdx.x == 0) report_status(4 /* SSM_ERR_BAD_SLOT */);
      continue;
    }
    float part = 0.f, uval = 0.f;
    if (valid) {
      const T *xu = static_cast<const T *>(args.u) + r * args.x_stride + d;
      const T *xd = static_cast<const T *>(args.delta) + r * args.x_stride + d;
      uval = Elem<T>::to_f32(*xu);
      const float dt = softplus_t<kFast>(Elem<T>::to_f32(*xd) + (args.bias ? args.bias[d] : 0.f));
      const float dtu = dt * uval;
      float4 *hp = reinterpret_cast<float4 *>(args.pool + (slot * args.dim + d) * N + 4 * q);
      const float4 a4 = *reinterpret_cast<const float4 *>(args.A + int64_t(d) * N + 4 * q);
      const T *Bv = static_cast<const T *>(args.B) + r * args.bc_stride + 4 * q;
      const T *Cv = static_cast<const T *>(args.C) + r * args.bc_stride + 4 * q;
      const float4 h = *hp;
      float hv[4] = {h.x, h.y, h.z, h.w};
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float abar = ex2_approx(dt * av[k] * kLog2e);
        hv[k] = fmaf(abar, hv[k], dtu * Elem<T>::to_f32(Bv[k]));
        part = fmaf(Elem<T>::to_f32(Cv[k]), hv[k], part);
      }
      *hp = make_float4(hv[0], hv[1], hv[2], hv[3]);
    }
    // reduce over the Q lanes of this channel (aligned groups inside one warp)
    for (int off = 1; off < Q; off *= 2) part += __shfl_xor_sync(0xffffffffu, part, off);
    if (valid && q == 0) {
      float v = fmaf(args.Dskip ? args.Dskip[d] : 0.f, uval, part);
      if constexpr (HAS_Z) {
        const T *xz = static_cast<const T *>(args.z) + r * args.x_stride + d;
        v *= silu_t<kFast>(Elem<T>::to_f32(*xz));
      }
      static_cast<TO *>(args.y)[r * args.x_stride + d] = Elem<TO>::from_f32(v);
    }
  }
}

}  // namespace ssm
