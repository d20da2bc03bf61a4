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
// Lanes are interleaved: lane = seg * CPW + cg.  The CPW channel groups of an 8-lane
// shared-memory phase therefore read the same B/C words (broadcast), and the distinct
// segments of a phase hit distinct banks.
//
// Staging.  The u, delta, z rows of the tile and the B, C rows of the chunk window are copied
// into shared memory (double-buffered) while the previous chunk is computed: one TMA bulk
// copy per row (cp.async.bulk completing on an mbarrier) when every row is 16-byte aligned,
// element-wise loads otherwise.  B and C stay in the input dtype in shared memory (a bf16
// value is widened in a register when used), which halves their shared-memory traffic.
// u/delta/z rows are padded by 16 bytes so that the channel groups of a phase read
// different banks.  Chunks that lie entirely inside the sequence skip all masking.
//
// Windows start at the sequence start rounded down to a 16-byte boundary; steps outside
// [seq_start, seq_end) are made identities (Delta = 0, Delta*u = 0, B = 0) and are not
// stored, which also resets the state at packed-sequence boundaries ("ufo.work" §4.2).
#pragma once

#include <type_traits>

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

// Packed sequences are visited longest first (CTAs with low indices start first), which
// keeps the tail short when lengths differ; the ordering is computed in each CTA, so it is
// only done for modest sequence counts.
constexpr int kMaxSortedSeqs = 64;

template <typename T, int N, int KI, int SPW, int CPW, int WARPS>
struct ChunkCfg {
  static constexpr int kTC = SPW * KI;     // chunk length (time steps)
  static constexpr int kCT = CPW * WARPS;  // channels per CTA
  static constexpr int kVec = Elem<T>::kVec;
  static constexpr int kThreads = WARPS * 32;
  static constexpr int kXPitch = kTC + kVec;  // u/delta/z row pitch (elements): +16 bytes
  // shared memory layout (bytes), everything double-buffered except the parameters
  static constexpr size_t kXBytes = size_t(3) * kCT * kXPitch * sizeof(T);  // u, delta, z
  static constexpr size_t kBCBytes = size_t(2) * N * kTC * sizeof(T);       // B, C
  static constexpr size_t kParamBytes =
      size_t(2) * kCT * N * sizeof(float) + size_t(2) * kCT * sizeof(float) + kMaxSortedSeqs * sizeof(int);
  static constexpr size_t kSmemBytes = 2 * kXBytes + 2 * kBCBytes + kParamBytes;
  static_assert(KI % 4 == 0 && KI % kVec == 0, "a lane's steps must be whole 16-byte vectors");
  static_assert(32 % SPW == 0 && CPW * SPW == 32, "lane split");
  static_assert(kXBytes % 16 == 0 && kBCBytes % 16 == 0, "16-byte aligned buffers");
};

template <typename T, typename TO, int N, int KI, int SPW, int CPW, int WARPS, bool HAS_Z, bool VEC>
__global__ void __launch_bounds__(WARPS * 32, (WARPS <= 8 ? 16 / WARPS : 1))
chunk_scan_kernel(const ScanArgs args) {
  using Cfg = ChunkCfg<T, N, KI, SPW, CPW, WARPS>;
  constexpr int TC = Cfg::kTC, CT = Cfg::kCT, V = Cfg::kVec, NT = Cfg::kThreads, XP = Cfg::kXPitch;
  constexpr int LV = KI / V;  // 16-byte vectors per lane
  constexpr bool kFast = Elem<T>::kFast;
  constexpr size_t kXElems = Cfg::kXBytes / sizeof(T), kBCElems = Cfg::kBCBytes / sizeof(T);

  extern __shared__ __align__(16) unsigned char smem[];
  T *const xs0 = reinterpret_cast<T *>(smem);                          // [2][3][CT][XP]
  T *const bc0 = reinterpret_cast<T *>(smem + 2 * Cfg::kXBytes);       // [2][2][N][TC]
  float *A2s = reinterpret_cast<float *>(smem + 2 * Cfg::kXBytes + 2 * Cfg::kBCBytes);  // [CT][N]
  float *carry_s = A2s + CT * N;                                       // [CT][N]
  float *Dsk = carry_s + CT * N;                                       // [CT]
  float *bias_s = Dsk + CT;                                            // [CT]
  int *order = reinterpret_cast<int *>(bias_s + CT);                   // [kMaxSortedSeqs]
  __shared__ __align__(8) uint64_t bars[2];                           // chunk-arrival barriers

  const int tile = blockIdx.x % args.ntiles;
  int s = blockIdx.x / args.ntiles;
  const int d0 = tile * CT;
  int64_t t_lo, t_hi, xbase, bcbase;
  if (args.cu_seqlens) {
    if (args.nseq <= kMaxSortedSeqs) {
      // rank sequences by length (descending, ties by index); order[rank] = sequence
      for (int i = threadIdx.x; i < args.nseq; i += NT) {
        const int li = args.cu_seqlens[i + 1] - args.cu_seqlens[i];
        int rank = 0;
        for (int j = 0; j < args.nseq; ++j) {
          const int lj = args.cu_seqlens[j + 1] - args.cu_seqlens[j];
          rank += (lj > li) || (lj == li && j < i);
        }
        order[rank] = i;
      }
      __syncthreads();
      s = order[s];
    }
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

  // tensor bases are read from the kernel parameters where used
#define SSM_GU static_cast<const T *>(args.u)
#define SSM_GDL static_cast<const T *>(args.delta)
#define SSM_GZ static_cast<const T *>(args.z)
#define SSM_GB static_cast<const T *>(args.B)
#define SSM_GC static_cast<const T *>(args.C)
  constexpr int nx = HAS_Z ? 3 : 2;
  const int nvalid_ch = int(min64(CT, args.dim - d0));
  // rows are readable up to the seqlen rounded up to a 16-byte vector (row strides are
  // multiples of 16 bytes on this path)
  const int64_t seqlen_r = (args.seqlen + V - 1) / V * V;

  // TMA: chunk c's u/delta/z and B/C rows into buffer `buf`.
  auto issue_chunk = [&](int buf, int c) {
    const int64_t wstart = w0 + int64_t(c) * TC;
    const int64_t wend = min64(wstart + TC, seqlen_r);
    const uint32_t row_bytes = uint32_t((wend - wstart) * int64_t(sizeof(T)));
    T *xdst = xs0 + buf * kXElems;
    T *bdst = bc0 + buf * kBCElems;
    fence_proxy_async_smem();
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&bars[buf], row_bytes * uint32_t(nx * nvalid_ch + 2 * N));
    for (int r = threadIdx.x; r < nx * CT + 2 * N; r += NT) {
      if (r < nx * CT) {
        const int which = r / CT, ch = r % CT;
        if (ch >= nvalid_ch) continue;
        const T *base = which == 0 ? SSM_GU : (which == 1 ? SSM_GDL : SSM_GZ);
        bulk_g2s(xdst + size_t(r) * XP, base + xbase + (d0 + ch) * args.x_dim_stride + wstart, row_bytes,
                 &bars[buf]);
      } else {
        const int r2 = r - nx * CT, which = r2 / N, n = r2 % N;
        const T *base = which == 0 ? SSM_GB : SSM_GC;
        bulk_g2s(bdst + size_t(r2) * TC, base + bcbase + int64_t(n) * args.bc_state_stride + wstart, row_bytes,
                 &bars[buf]);
      }
    }
  };
  // Element-wise staging for rows that are not 16-byte aligned (zero outside the tensor).
  auto stage_scalar = [&](int buf, int c) {
    T *xdst = xs0 + buf * kXElems;
    T *bdst = bc0 + buf * kBCElems;
    const int64_t wstart = w0 + int64_t(c) * TC;
    for (int i = threadIdx.x; i < nx * CT * TC; i += NT) {
      const int row = i / TC, j = i % TC;
      const int which = row / CT, ch = row % CT;
      const int64_t d = d0 + ch, t = wstart + j;
      const T *base = which == 0 ? SSM_GU : (which == 1 ? SSM_GDL : SSM_GZ);
      T val = Elem<T>::from_f32(0.f);
      if (d < args.dim && t < args.seqlen) val = base[xbase + d * args.x_dim_stride + t];
      xdst[size_t(row) * XP + j] = val;
    }
    for (int i = threadIdx.x; i < 2 * N * TC; i += NT) {
      const int row = i / TC, j = i % TC;
      const int which = row / N, n = row % N;
      const int64_t t = wstart + j;
      const T *base = which == 0 ? SSM_GB : SSM_GC;
      T val = Elem<T>::from_f32(0.f);
      if (t < args.seqlen) val = base[bcbase + int64_t(n) * args.bc_state_stride + t];
      bdst[size_t(row) * TC + j] = val;
    }
  };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cg = lane % CPW, seg = lane / CPW;  // interleaved channel groups
  const int ch = warp * CPW + cg;
  const int64_t d = d0 + ch;
  const bool ch_ok = d < args.dim;

  if constexpr (VEC) {
    if (threadIdx.x == 0) {
      mbar_init(&bars[0], 1);
      mbar_init(&bars[1], 1);
      mbar_init_fence();
    }
    __syncthreads();
    if (nchunks > 0) issue_chunk(0, 0);
  }

  // One chunk of the lane's work; the masked instance handles chunks that straddle a
  // sequence end.
  auto compute_chunk = [&](auto masked_tag, const T *X, const T *Bsm, const T *Csm, int64_t wstart, int rel_lo,
                           int rel_hi) {
    constexpr bool kMasked = decltype(masked_tag)::value;
    const int tl0 = seg * KI;  // chunk-local first step of this lane
    // ---- prologue: Delta and Delta*u for the lane's KI steps (as pairs of steps) ----
    constexpr int KP = KI / 2;
    float2 dl[KP], du[KP], y[KP];
    float dsum = 0.f;
    {
      const T *ru = X + size_t(ch) * XP + tl0;
      const T *rd = X + size_t(CT + ch) * XP + tl0;
      const float bias = bias_s[ch];
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        float2 vu[V / 2], vd[V / 2];
        unpack16x2<T>(*reinterpret_cast<const uint4 *>(ru + lv * V), vu);
        unpack16x2<T>(*reinterpret_cast<const uint4 *>(rd + lv * V), vd);
#pragma unroll
        for (int e = 0; e < V / 2; ++e) {
          const int p = lv * (V / 2) + e;
          float2 dt = make_float2(softplus_t<kFast>(vd[e].x + bias), softplus_t<kFast>(vd[e].y + bias));
          if constexpr (kMasked) {
            const int i = tl0 + 2 * p;
            dt.x = (i >= rel_lo && i < rel_hi) ? dt.x : 0.f;
            dt.y = (i + 1 >= rel_lo && i + 1 < rel_hi) ? dt.y : 0.f;
            // select, so a non-finite u outside the sequence stays out
            du[p] = make_float2(dt.x != 0.f ? dt.x * vu[e].x : 0.f, dt.y != 0.f ? dt.y * vu[e].y : 0.f);
          } else {
            du[p] = __fmul2_rn(dt, vu[e]);
          }
          dl[p] = dt;
          dsum += dt.x + dt.y;
          y[p] = make_float2(0.f, 0.f);
        }
      }
    }

    // ---- state loop ----
#pragma unroll 1
    for (int n = 0; n < N; ++n) {
      const float A2 = A2s[ch * N + n];
      const float2 A22 = make_float2(A2, A2);
      const float carry = carry_s[ch * N + n];
      float a[KI];
      float2 b[KP];
      float G = 0.f;
      const T *rb = Bsm + size_t(n) * TC + tl0;
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        float2 bb[V / 2];
        unpack16x2<T>(*reinterpret_cast<const uint4 *>(rb + lv * V), bb);
#pragma unroll
        for (int e = 0; e < V / 2; ++e) {
          const int p = lv * (V / 2) + e;
          const float2 x = __fmul2_rn(dl[p], A22);
          a[2 * p] = ex2_approx(x.x);
          a[2 * p + 1] = ex2_approx(x.y);
          if constexpr (kMasked) {
            // stale B outside the window never reaches h (du is 0 there, B may be non-finite)
            b[p] = make_float2(du[p].x != 0.f ? du[p].x * bb[e].x : 0.f, du[p].y != 0.f ? du[p].y * bb[e].y : 0.f);
          } else {
            b[p] = __fmul2_rn(du[p], bb[e]);
          }
          G = fmaf(a[2 * p], G, b[p].x);
          G = fmaf(a[2 * p + 1], G, b[p].y);
        }
      }
      float P = ex2_approx(dsum * A2);  // product of the lane's a_i
      // inclusive scan of segment operators across the SPW segment lanes of this channel
#pragma unroll
      for (int off = 1; off < SPW; off *= 2) {
        const float Pu = __shfl_up_sync(0xffffffffu, P, off * CPW);
        const float Gu = __shfl_up_sync(0xffffffffu, G, off * CPW);
        if (seg >= off) {
          G = fmaf(P, Gu, G);
          P *= Pu;
        }
      }
      float Pe = __shfl_up_sync(0xffffffffu, P, CPW);
      float Ge = __shfl_up_sync(0xffffffffu, G, CPW);
      if (seg == 0) {
        Pe = 1.f;
        Ge = 0.f;
      }
      float h = fmaf(Pe, carry, Ge);  // state entering this lane's first step
      __syncwarp();
      if (seg == SPW - 1) carry_s[ch * N + n] = fmaf(P, carry, G);  // state leaving the chunk
      const T *rc = Csm + size_t(n) * TC + tl0;
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        float2 cc[V / 2];
        unpack16x2<T>(*reinterpret_cast<const uint4 *>(rc + lv * V), cc);
#pragma unroll
        for (int e = 0; e < V / 2; ++e) {
          const int p = lv * (V / 2) + e;
          float2 hh;
          h = fmaf(a[2 * p], h, b[p].x);
          hh.x = h;
          h = fmaf(a[2 * p + 1], h, b[p].y);
          hh.y = h;
          y[p] = __ffma2_rn(cc[e], hh, y[p]);
        }
      }
    }

    // ---- epilogue: skip term, gate, store ----
    if (ch_ok) {
      const float Dd = Dsk[ch];
      const T *ru = X + size_t(ch) * XP + tl0;
      [[maybe_unused]] const T *rz = X + size_t(2 * CT + ch) * XP + tl0;
      constexpr int VO = Elem<TO>::kVec;  // output elements per 16-byte store
      float yo[KI];
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        float vu[V];
        [[maybe_unused]] float vz[V];
        unpack16<T>(*reinterpret_cast<const uint4 *>(ru + lv * V), vu);
        if constexpr (HAS_Z) unpack16<T>(*reinterpret_cast<const uint4 *>(rz + lv * V), vz);
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const int i = lv * V + e;
          float v = fmaf(Dd, vu[e], (i & 1) ? y[i / 2].y : y[i / 2].x);
          if constexpr (HAS_Z) v *= silu_t<kFast>(vz[e]);
          yo[i] = v;
        }
      }
      TO *gy = static_cast<TO *>(args.y) + xbase + d * args.x_dim_stride + wstart + tl0;
      if (VEC && (!kMasked || (tl0 >= rel_lo && tl0 + KI <= rel_hi))) {
#pragma unroll
        for (int v = 0; v < KI / VO; ++v) *reinterpret_cast<uint4 *>(gy + v * VO) = pack16<TO>(yo + v * VO);
      } else {
#pragma unroll
        for (int i = 0; i < KI; ++i)
          if (!kMasked || (tl0 + i >= rel_lo && tl0 + i < rel_hi)) gy[i] = Elem<TO>::from_f32(yo[i]);
      }
    }
  };

  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    const int64_t wstart = w0 + int64_t(c) * TC;
    if constexpr (VEC) {
      mbar_wait_bounded(&bars[buf], uint32_t(c >> 1) & 1u);
    } else {
      stage_scalar(buf, c);
    }
    __syncthreads();  // chunk c visible to all; everyone is done with chunk c-1's buffers
    if constexpr (VEC) {
      if (c + 1 < nchunks) issue_chunk(buf ^ 1, c + 1);  // streams in while chunk c is computed
    }
    // chunk-relative sequence bounds; a chunk strictly inside the sequence needs no masks
    const int rel_lo = int(max64(t_lo - wstart, -1));
    const int rel_hi = int(min64(t_hi - wstart, TC + 1));
    const T *X = xs0 + buf * kXElems;
    const T *Bsm = bc0 + buf * kBCElems;
    const T *Csm = Bsm + size_t(N) * TC;
    if (rel_lo <= 0 && rel_hi >= TC)
      compute_chunk(std::false_type{}, X, Bsm, Csm, wstart, rel_lo, rel_hi);
    else
      compute_chunk(std::true_type{}, X, Bsm, Csm, wstart, rel_lo, rel_hi);
  }
#undef SSM_GU
#undef SSM_GDL
#undef SSM_GZ
#undef SSM_GB
#undef SSM_GC

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
