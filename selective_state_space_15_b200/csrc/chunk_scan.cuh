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
// Staging.  u, delta, z rows of the tile (double-buffered) and the B, C rows of the chunk
// window (single buffer, consumed right after arrival) are copied into shared memory while
// the previous chunk is computed: one TMA bulk copy per row (cp.async.bulk completing on an
// mbarrier) when every row is 16-byte aligned, element-wise loads otherwise.  B and C are
// converted once per chunk to float32 in an interleaved [n][KI/4][SPW] float4 layout: the
// SPW segment lanes read consecutive 16-byte words and the CPW channel groups of a warp
// read the same words.  Chunks that lie entirely inside the sequence skip all masking.
//
// Windows start at the sequence start rounded down to a 16-byte boundary; steps outside
// [seq_start, seq_end) are made identities (Delta = 0, Delta*u = 0, B = C = 0) and are not
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
  static constexpr int kVPR = kTC / kVec;  // 16-byte vectors per staged row
  // shared memory layout (bytes)
  static constexpr size_t kXBytes = size_t(3) * kCT * kTC * sizeof(T);  // u, delta, z of one chunk
  static constexpr size_t kBCRawBytes = size_t(2) * N * kTC * sizeof(T);
  static constexpr size_t kConvBytes = size_t(2) * N * kTC * sizeof(float);
  static constexpr size_t kParamBytes =
      size_t(2) * kCT * N * sizeof(float) + size_t(2) * kCT * sizeof(float) + kMaxSortedSeqs * sizeof(int);
  static constexpr size_t kSmemBytes = 2 * kXBytes + kBCRawBytes + kConvBytes + kParamBytes;
  static_assert(KI % 4 == 0 && KI % kVec == 0, "a lane's steps must be whole float4 and 16-byte vectors");
  static_assert(32 % SPW == 0 && CPW * SPW == 32, "lane split");
};


template <typename T, typename TO, int N, int KI, int SPW, int CPW, int WARPS, bool HAS_Z, bool VEC>
__global__ void __launch_bounds__(WARPS * 32, (WARPS <= 8 ? 16 / WARPS : 1))
chunk_scan_kernel(const ScanArgs args) {
  using Cfg = ChunkCfg<T, N, KI, SPW, CPW, WARPS>;
  constexpr int TC = Cfg::kTC, CT = Cfg::kCT, V = Cfg::kVec, NT = Cfg::kThreads, VPR = Cfg::kVPR;
  constexpr int LV = KI / V;  // 16-byte vectors per lane
  constexpr bool kFast = Elem<T>::kFast;

  extern __shared__ __align__(16) unsigned char smem[];
  T *const xs0 = reinterpret_cast<T *>(smem);  // u, delta, z rows; buffer b at xs0 + b * kXElems
  constexpr size_t kXElems = Cfg::kXBytes / sizeof(T);
  T *bcraw = reinterpret_cast<T *>(smem + 2 * Cfg::kXBytes);
  float4 *Bs4 = reinterpret_cast<float4 *>(smem + 2 * Cfg::kXBytes + Cfg::kBCRawBytes);  // [N][KI/4][SPW]
  float4 *Cs4 = Bs4 + N * (TC / 4);
  float *A2s = reinterpret_cast<float *>(Cs4 + N * (TC / 4));  // [CT][N]  A * log2(e)
  float *carry_s = A2s + CT * N;                                // [CT][N]
  float *Dsk = carry_s + CT * N;                                // [CT]
  float *bias_s = Dsk + CT;                                     // [CT]
  int *order = reinterpret_cast<int *>(bias_s + CT);            // [kMaxSortedSeqs]

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

  // tensor bases are read from the kernel parameters where used (no registers held across
  // the chunk loop)
#define SSM_GU static_cast<const T *>(args.u)
#define SSM_GDL static_cast<const T *>(args.delta)
#define SSM_GZ static_cast<const T *>(args.z)
#define SSM_GB static_cast<const T *>(args.B)
#define SSM_GC static_cast<const T *>(args.C)
  constexpr int nx = HAS_Z ? 3 : 2;

  __shared__ __align__(8) uint64_t bars[2];  // chunk-arrival barriers of the two X buffers
  const int nvalid_ch = int(min64(CT, args.dim - d0));
  // rows are readable up to the seqlen rounded up to a 16-byte vector (row strides are
  // multiples of 16 bytes on this path)
  const int64_t seqlen_r = (args.seqlen + V - 1) / V * V;

  // TMA: chunk c's u/delta/z rows into X buffer `buf` and its B/C rows into bcraw.
  auto issue_chunk = [&](int buf, int c) {
    const int64_t wstart = w0 + int64_t(c) * TC;
    const int64_t wend = min64(wstart + TC, seqlen_r);
    const uint32_t row_bytes = uint32_t((wend - wstart) * int64_t(sizeof(T)));
    T *xdst = xs0 + buf * kXElems;
    fence_proxy_async_smem();
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&bars[buf], row_bytes * uint32_t(nx * nvalid_ch + 2 * N));
    for (int r = threadIdx.x; r < nx * CT + 2 * N; r += NT) {
      if (r < nx * CT) {
        const int which = r / CT, ch = r % CT;
        if (ch >= nvalid_ch) continue;
        const T *base = which == 0 ? SSM_GU : (which == 1 ? SSM_GDL : SSM_GZ);
        bulk_g2s(xdst + size_t(r) * TC, base + xbase + (d0 + ch) * args.x_dim_stride + wstart, row_bytes,
                 &bars[buf]);
      } else {
        const int r2 = r - nx * CT, which = r2 / N, n = r2 % N;
        const T *base = which == 0 ? SSM_GB : SSM_GC;
        bulk_g2s(bcraw + size_t(r2) * TC, base + bcbase + int64_t(n) * args.bc_state_stride + wstart, row_bytes,
                 &bars[buf]);
      }
    }
  };
  // Element-wise staging (rows not 16-byte aligned): u/delta/z rows into xs[buf], B/C into bcraw.
  auto stage_scalar = [&](int buf, int c) {
    T *dst = xs0 + buf * kXElems;
    const int64_t wstart = w0 + int64_t(c) * TC;
    for (int i = threadIdx.x; i < nx * CT * TC; i += NT) {
      const int row = i / TC, j = i % TC;
      const int which = row / CT, ch = row % CT;
      const int64_t d = d0 + ch, t = wstart + j;
      const T *base = which == 0 ? SSM_GU : (which == 1 ? SSM_GDL : SSM_GZ);
      T val = Elem<T>::from_f32(0.f);
      if (d < args.dim && t < args.seqlen) val = base[xbase + d * args.x_dim_stride + t];
      dst[size_t(row) * TC + j] = val;
    }
    for (int i = threadIdx.x; i < 2 * N * TC; i += NT) {
      const int row = i / TC, j = i % TC;
      const int which = row / N, n = row % N;
      const int64_t t = wstart + j;
      const T *base = which == 0 ? SSM_GB : SSM_GC;
      T val = Elem<T>::from_f32(0.f);
      if (t < args.seqlen) val = base[bcbase + int64_t(n) * args.bc_state_stride + t];
      bcraw[size_t(row) * TC + j] = val;
    }
  };

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int cg = lane / SPW, seg = lane % SPW;
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

  for (int c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    const int64_t wstart = w0 + int64_t(c) * TC;
    if constexpr (VEC) {
      mbar_wait_bounded(&bars[buf], uint32_t(c >> 1) & 1u);
    } else {
      stage_scalar(buf, c);
    }
    __syncthreads();  // chunk c visible to all; everyone is done with chunk c-1
    // chunk-relative sequence bounds; a chunk strictly inside the sequence needs no masks
    const int rel_lo = int(max64(t_lo - wstart, -1));
    const int rel_hi = int(min64(t_hi - wstart, TC + 1));
    const bool full = rel_lo <= 0 && rel_hi >= TC;

    // B, C -> float32 interleaved layout (steps outside the sequence zeroed).
    auto convert = [&](auto masked_tag) {
      constexpr bool kMasked = decltype(masked_tag)::value;
      for (int i = threadIdx.x; i < 2 * N * VPR; i += NT) {
        const int row = i / VPR, v = i % VPR;  // row < N: B, else C
        const int n = row % N;
        float4 *dstv = row < N ? Bs4 : Cs4;
        float raw[V];
        unpack16<T>(*reinterpret_cast<const uint4 *>(bcraw + size_t(row) * TC + v * V), raw);
#pragma unroll
        for (int g = 0; g < V / 4; ++g) {
          const int tl = v * V + g * 4;  // chunk-local step of the first of 4
          const int sg = tl / KI, q = (tl % KI) / 4;
          float f[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) f[r] = (!kMasked || (tl + r >= rel_lo && tl + r < rel_hi)) ? raw[g * 4 + r] : 0.f;
          dstv[(n * (KI / 4) + q) * SPW + sg] = make_float4(f[0], f[1], f[2], f[3]);
        }
      }
    };
    if (full) convert(std::false_type{});
    else convert(std::true_type{});
    __syncthreads();  // conversions visible; bcraw free again

    // stream chunk c+1 in while chunk c is computed
    if constexpr (VEC) {
      if (c + 1 < nchunks) issue_chunk(buf ^ 1, c + 1);
    }

    const T *X = xs0 + buf * kXElems;
    // ---- per-lane prologue: Delta and Delta*u for the lane's KI steps ----
    float dl[KI], du[KI], y[KI];
    float dsum = 0.f;
    {
      const T *ru = X + size_t(ch) * TC;
      const T *rd = X + size_t(CT + ch) * TC;
      const float bias = bias_s[ch];
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        const int pv = (seg * LV + lv) * V;
        float vu[V], vd[V];
        unpack16<T>(*reinterpret_cast<const uint4 *>(ru + pv), vu);
        unpack16<T>(*reinterpret_cast<const uint4 *>(rd + pv), vd);
        if (full) {
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const int i = lv * V + e;
            dl[i] = softplus_t<kFast>(vd[e] + bias);
            du[i] = dl[i] * vu[e];
          }
        } else {
#pragma unroll
          for (int e = 0; e < V; ++e) {
            const int i = lv * V + e;
            const int tl = seg * KI + i;
            const bool in = tl >= rel_lo && tl < rel_hi;
            const float dt = softplus_t<kFast>(vd[e] + bias);
            dl[i] = in ? dt : 0.f;
            du[i] = in ? dt * vu[e] : 0.f;  // select, so a non-finite u outside the sequence stays out
          }
        }
#pragma unroll
        for (int e = 0; e < V; ++e) {
          dsum += dl[lv * V + e];
          y[lv * V + e] = 0.f;
        }
      }
    }

    // ---- state loop ----
#pragma unroll 1
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
      const T *ru = X + size_t(ch) * TC;
      const T *rz = X + size_t(2 * CT + ch) * TC;
      const int64_t t0 = wstart + seg * KI;
      constexpr int VO = Elem<TO>::kVec;  // output elements per 16-byte store
#pragma unroll
      for (int lv = 0; lv < LV; ++lv) {
        const int pv = (seg * LV + lv) * V;
        float vu[V], vz[V];
        unpack16<T>(*reinterpret_cast<const uint4 *>(ru + pv), vu);
        if constexpr (HAS_Z) unpack16<T>(*reinterpret_cast<const uint4 *>(rz + pv), vz);
#pragma unroll
        for (int e = 0; e < V; ++e) {
          const int i = lv * V + e;
          float v = fmaf(Dd, vu[e], y[i]);
          if constexpr (HAS_Z) v *= silu_t<kFast>(vz[e]);
          y[i] = v;
        }
      }
      TO *gy = static_cast<TO *>(args.y) + xbase + d * args.x_dim_stride + t0;
      const int tl0 = seg * KI;
      if (VEC && tl0 >= rel_lo && tl0 + KI <= rel_hi) {
#pragma unroll
        for (int v = 0; v < KI / VO; ++v) *reinterpret_cast<uint4 *>(gy + v * VO) = pack16<TO>(y + v * VO);
      } else {
#pragma unroll
        for (int i = 0; i < KI; ++i)
          if (tl0 + i >= rel_lo && tl0 + i < rel_hi) gy[i] = Elem<TO>::from_f32(y[i]);
      }
    }
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
