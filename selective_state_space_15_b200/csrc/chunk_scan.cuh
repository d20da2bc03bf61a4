// Chunked selective-scan kernel (prefill, fixed-length and packed varlen).
//
// Work decomposition.  A CTA owns one (sequence, tile of CT channels) pair and walks the
// sequence in chunks of TC = SPW * KI time steps, carrying the per-(channel, state) state
// across chunks in shared memory ("ufo.work" page, §3.1: h_end = Abar_chunk h_start +
// Bbar_chunk).  Inside a chunk a warp holds CPW channels x SPW time segments; each lane
// owns KI consecutive steps of one channel.  For every state n the lane
//   1. forms a_i = exp(Delta_i A[d,n]) and b_i = Delta_i B_i[n] u_i for its KI steps and
//      folds them into its segment operator (P, G) with h_end = P h_start + G,
//   2. composes the operators of the SPW segments with a Kogge-Stone warp scan
//      (the same associative pair composition as the chunk operators),
//   3. re-walks its steps from the exclusive prefix applied to the chunk carry, producing
//      h_t and accumulating y_t += C_t[n] h_t in registers.
// No h_t ever leaves registers; only y and the final state are written.  Each exponential
// exp(Delta A) is evaluated once.
//
// Staging.  u, delta, z rows of the tile and the B, C rows of the chunk window are copied
// into shared memory with 16-byte cp.async (double-buffered: chunk c+1 streams in while
// chunk c is computed).  B and C are then converted to float32 in an interleaved layout
// [n][KI/4][SPW] of float4 so that the SPW segment lanes read consecutive 16-byte words
// (no bank conflicts) and the CPW channel groups of a warp read the same words (broadcast).
//
// Windows start at the sequence start rounded down to a 16-byte boundary; steps outside
// [seq_start, seq_end) are made identities (Delta = 0, Delta*u = 0, B = C = 0) and are not
// stored, which also resets the state at packed-sequence boundaries ("ufo.work" §4.2).
#pragma once

#include "common.cuh"

namespace ssm {

struct ScanArgs {
  const void *u, *delta, *z, *B, *C;
  const float *A, *Dskip, *bias, *h0;
  void *y;
  float *h_last;
  const int32_t *cu_seqlens;  // nullptr: fixed-length batch
  int64_t dim, seqlen;
  int64_t x_batch_stride, x_dim_stride, bc_batch_stride, bc_state_stride;
  int nseq;    // sequences (batch size or number of packed sequences)
  int ntiles;  // channel tiles per sequence
};

template <typename T, int N, int KI, int SPW, int CPW, int WARPS>
struct ChunkCfg {
  static constexpr int kTC = SPW * KI;     // chunk length (time steps)
  static constexpr int kCT = CPW * WARPS;  // channels per CTA
  static constexpr int kVec = Elem<T>::kVec;
  static constexpr int kThreads = WARPS * 32;
  // shared memory layout (bytes)
  static constexpr size_t kXBytes = size_t(3) * kCT * kTC * sizeof(T);  // u, delta, z
  static constexpr size_t kBCRawBytes = size_t(2) * N * kTC * sizeof(T);
  static constexpr size_t kStageBytes = kXBytes + kBCRawBytes;
  static constexpr size_t kConvBytes = size_t(2) * N * kTC * sizeof(float);
  static constexpr size_t kParamBytes = size_t(2) * kCT * N * sizeof(float) + size_t(2) * kCT * sizeof(float);
  static constexpr size_t kSmemBytes = 2 * kStageBytes + kConvBytes + kParamBytes;
  static_assert(KI % 4 == 0 && KI % kVec == 0, "a lane's steps must be whole float4 and 16-byte vectors");
  static_assert(kTC % kVec == 0, "chunk must be whole vectors");
  static_assert(32 % SPW == 0 && CPW * SPW == 32, "lane split");
};

template <typename T, typename TO, int N, int KI, int SPW, int CPW, int WARPS, bool HAS_Z, bool VEC>
__global__ void __launch_bounds__(WARPS * 32)
chunk_scan_kernel(const ScanArgs args) {
  using Cfg = ChunkCfg<T, N, KI, SPW, CPW, WARPS>;
  constexpr int TC = Cfg::kTC, CT = Cfg::kCT, V = Cfg::kVec, NT = Cfg::kThreads;
  constexpr bool kFast = Elem<T>::kFast;

  extern __shared__ __align__(16) unsigned char smem[];
  T *stage[2];
  stage[0] = reinterpret_cast<T *>(smem);
  stage[1] = reinterpret_cast<T *>(smem + Cfg::kStageBytes);
  float4 *Bs4 = reinterpret_cast<float4 *>(smem + 2 * Cfg::kStageBytes);  // [N][KI/4][SPW]
  float4 *Cs4 = Bs4 + N * (TC / 4);
  float *A2s = reinterpret_cast<float *>(Cs4 + N * (TC / 4));  // [CT][N]  A * log2(e)
  float *carry_s = A2s + CT * N;                                // [CT][N]
  float *Dsk = carry_s + CT * N;                                // [CT]
  float *bias_s = Dsk + CT;                                     // [CT]

  const int tile = blockIdx.x % args.ntiles;
  const int s = blockIdx.x / args.ntiles;
  const int d0 = tile * CT;
  int64_t t_lo, t_hi, xbase, bcbase;
  if (args.cu_seqlens) {
    t_lo = args.cu_seqlens[s];
    t_hi = args.cu_seqlens[s + 1];
    xbase = 0;
    bcbase = 0;
  } else {
    t_lo = 0;
    t_hi = args.seqlen;
    xbase = int64_t(s) * args.x_batch_stride;
    bcbase = int64_t(s) * args.bc_batch_stride;
  }
  const int64_t w0 = t_lo & ~int64_t(V - 1);
  const int nchunks = t_hi > t_lo ? int((t_hi - w0 + TC - 1) / TC) : 0;

  // per-tile constants and initial state
  for (int i = threadIdx.x; i < CT * N; i += NT) {
    const int ch = i / N, n = i % N;
    const int64_t d = d0 + ch;
    const bool ok = d < args.dim;
    A2s[i] = ok ? args.A[d * N + n] * kLog2e : 0.f;
    carry_s[i] = (ok && args.h0) ? args.h0[(int64_t(s) * args.dim + d) * N + n] : 0.f;
  }
  for (int i = threadIdx.x; i < CT; i += NT) {
    const int64_t d = d0 + i;
    const bool ok = d < args.dim;
    Dsk[i] = (ok && args.Dskip) ? args.Dskip[d] : 0.f;
    bias_s[i] = (ok && args.bias) ? args.bias[d] : 0.f;
  }

  const T *gu = static_cast<const T *>(args.u);
  const T *gdl = static_cast<const T *>(args.delta);
  const T *gz = static_cast<const T *>(args.z);
  const T *gB = static_cast<const T *>(args.B);
  const T *gC = static_cast<const T *>(args.C);

  // Stage chunk `c` into buffer `buf`: rows [x: 3*CT][bc: 2*N], TC elements each.
  auto stage_chunk = [&](int buf, int c) {
    T *dst = stage[buf];
    const int64_t wstart = w0 + int64_t(c) * TC;
    constexpr int nx = HAS_Z ? 3 : 2;
    constexpr int rows = nx * CT + 2 * N;
    if constexpr (VEC) {
      constexpr int vpr = TC / V;  // vectors per row
      for (int i = threadIdx.x; i < rows * vpr; i += NT) {
        const int row = i / vpr, v = i % vpr;
        const int64_t t = wstart + int64_t(v) * V;
        const T *base, *src;
        int64_t lim;
        T *sdst;
        if (row < nx * CT) {
          const int which = row / CT, ch = row % CT;
          const int64_t d = d0 + ch;
          base = which == 0 ? gu : (which == 1 ? gdl : gz);
          lim = d < args.dim ? args.seqlen : 0;
          src = base + (d < args.dim ? xbase + d * args.x_dim_stride + t : 0);
          sdst = dst + (size_t(which) * CT + ch) * TC + v * V;
        } else {
          const int r2 = row - nx * CT, which = r2 / N, n = r2 % N;
          base = which == 0 ? gB : gC;
          lim = args.seqlen;
          src = base + bcbase + int64_t(n) * args.bc_state_stride + t;
          sdst = dst + size_t(3) * CT * TC + (size_t(which) * N + n) * TC + v * V;
        }
        int64_t avail = lim - t;
        avail = avail < 0 ? 0 : (avail > V ? V : avail);
        // a zero-byte copy reads nothing; point it at the tensor base all the same
        cp_async_16(sdst, avail > 0 ? (const void *)src : (const void *)base, int(avail * sizeof(T)));
      }
    } else {
      for (int i = threadIdx.x; i < rows * TC; i += NT) {
        const int row = i / TC, j = i % TC;
        const int64_t t = wstart + j;
        T val = Elem<T>::from_f32(0.f);
        T *sdst;
        if (row < nx * CT) {
          const int which = row / CT, ch = row % CT;
          const int64_t d = d0 + ch;
          const T *base = which == 0 ? gu : (which == 1 ? gdl : gz);
          if (d < args.dim && t < args.seqlen) val = base[xbase + d * args.x_dim_stride + t];
          sdst = dst + (size_t(which) * CT + ch) * TC + j;
        } else {
          const int r2 = row - nx * CT, which = r2 / N, n = r2 % N;
          const T *base = which == 0 ? gB : gC;
          if (t < args.seqlen) val = base[bcbase + int64_t(n) * args.bc_state_stride + t];
          sdst = dst + size_t(3) * CT * TC + (size_t(which) * N + n) * TC + j;
        }
        *sdst = val;
      }
    }
  };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cg = lane / SPW, seg = lane % SPW;
  const int ch = warp * CPW + cg;
  const int64_t d = d0 + ch;
  const bool ch_ok = d < args.dim;

  if constexpr (VEC) {
    if (nchunks > 0) stage_chunk(0, 0);
    cp_async_commit();
  }

  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    const int64_t wstart = w0 + int64_t(c) * TC;
    if constexpr (VEC) {
      cp_async_wait_all();
      __syncthreads();  // chunk c visible; everyone is done with chunk c-1
      if (c + 1 < nchunks) stage_chunk(buf ^ 1, c + 1);
      cp_async_commit();
    } else {
      __syncthreads();  // everyone is done with chunk c-1's buffers
      stage_chunk(buf, c);
      __syncthreads();
    }
    const T *X = stage[buf];
    const T *Braw = X + size_t(3) * CT * TC;
    const T *Craw = Braw + size_t(N) * TC;

    // B, C -> float32 interleaved layout, steps outside the sequence zeroed.
    for (int i = threadIdx.x; i < N * (TC / 4); i += NT) {
      const int sg = i % SPW, q = (i / SPW) % (KI / 4), n = i / (SPW * (KI / 4));
      const int tl = sg * KI + q * 4;
      float bv[4], cv[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t tg = wstart + tl + r;
        const bool in = tg >= t_lo && tg < t_hi;
        bv[r] = in ? Elem<T>::to_f32(Braw[size_t(n) * TC + tl + r]) : 0.f;
        cv[r] = in ? Elem<T>::to_f32(Craw[size_t(n) * TC + tl + r]) : 0.f;
      }
      Bs4[i] = make_float4(bv[0], bv[1], bv[2], bv[3]);
      Cs4[i] = make_float4(cv[0], cv[1], cv[2], cv[3]);
    }
    __syncthreads();

    // ---- per-lane prologue: Delta and Delta*u for the lane's KI steps ----
    const T *xu = X + size_t(ch) * TC + seg * KI;
    const T *xd = X + size_t(CT + ch) * TC + seg * KI;
    const float bias = bias_s[ch];
    float dl[KI], du[KI], y[KI];
    float dsum = 0.f;
#pragma unroll
    for (int i = 0; i < KI; ++i) {
      const int64_t tg = wstart + seg * KI + i;
      const bool in = tg >= t_lo && tg < t_hi;
      const float dt = softplus_t<kFast>(Elem<T>::to_f32(xd[i]) + bias);
      dl[i] = in ? dt : 0.f;
      du[i] = in ? dt * Elem<T>::to_f32(xu[i]) : 0.f;
      dsum += dl[i];
      y[i] = 0.f;
    }

    // ---- state loop ----
#pragma unroll 2
    for (int n = 0; n < N; ++n) {
      const float A2 = A2s[ch * N + n];
      const float carry = carry_s[ch * N + n];
      float a[KI], b[KI];
      float G = 0.f;
#pragma unroll
      for (int q = 0; q < KI / 4; ++q) {
        const float4 bq = Bs4[(n * (KI / 4) + q) * SPW + seg];
        const float bb[4] = {bq.x, bq.y, bq.z, bq.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = q * 4 + r;
          a[i] = ex2_approx(dl[i] * A2);
          b[i] = du[i] * bb[r];
          G = fmaf(a[i], G, b[i]);
        }
      }
      float P = ex2_approx(dsum * A2);  // product of the lane's a_i
      // inclusive scan of segment operators across the SPW lanes of this channel
#pragma unroll
      for (int off = 1; off < SPW; off *= 2) {
        const float Pu = __shfl_up_sync(0xffffffffu, P, off, SPW);
        const float Gu = __shfl_up_sync(0xffffffffu, G, off, SPW);
        if (seg >= off) {
          G = fmaf(P, Gu, G);
          P *= Pu;
        }
      }
      float Pe = __shfl_up_sync(0xffffffffu, P, 1, SPW);
      float Ge = __shfl_up_sync(0xffffffffu, G, 1, SPW);
      if (seg == 0) {
        Pe = 1.f;
        Ge = 0.f;
      }
      float h = fmaf(Pe, carry, Ge);  // state entering this lane's first step
      __syncwarp();
      if (seg == SPW - 1) carry_s[ch * N + n] = fmaf(P, carry, G);  // state leaving the chunk
#pragma unroll
      for (int q = 0; q < KI / 4; ++q) {
        const float4 cq = Cs4[(n * (KI / 4) + q) * SPW + seg];
        const float cc[4] = {cq.x, cq.y, cq.z, cq.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = q * 4 + r;
          h = fmaf(a[i], h, b[i]);
          y[i] = fmaf(cc[r], h, y[i]);
        }
      }
    }

    // ---- epilogue: skip term, gate, store ----
    if (ch_ok) {
      const float Dd = Dsk[ch];
      const T *xz = X + size_t(2 * CT + ch) * TC + seg * KI;
      const int64_t t0 = wstart + seg * KI;
      constexpr int VO = Elem<TO>::kVec;  // output elements per 16-byte store
      alignas(16) TO out[KI];
#pragma unroll
      for (int i = 0; i < KI; ++i) {
        float v = fmaf(Dd, Elem<T>::to_f32(xu[i]), y[i]);
        if constexpr (HAS_Z) v *= silu_t<kFast>(Elem<T>::to_f32(xz[i]));
        out[i] = Elem<TO>::from_f32(v);
      }
      TO *gy = static_cast<TO *>(args.y) + xbase + d * args.x_dim_stride + t0;
      if (VEC && t0 >= t_lo && t0 + KI <= t_hi) {
#pragma unroll
        for (int v = 0; v < KI / VO; ++v)
          *reinterpret_cast<uint4 *>(gy + v * VO) = *reinterpret_cast<const uint4 *>(out + v * VO);
      } else {
#pragma unroll
        for (int i = 0; i < KI; ++i)
          if (t0 + i >= t_lo && t0 + i < t_hi) gy[i] = out[i];
      }
    }
  }

  // final state of each channel of the tile
  __syncthreads();
  if (args.h_last) {
    for (int i = threadIdx.x; i < CT * N; i += NT) {
      const int c2 = i / N, n = i % N;
      const int64_t dd = d0 + c2;
      if (dd < args.dim) args.h_last[(int64_t(s) * args.dim + dd) * N + n] = carry_s[i];
    }
  }
}

}  // namespace ssm
