// Lane-sequential selective-scan kernel (prefill, fixed-length and packed varlen).
//
// Each lane owns one channel and NS = N / LPC of its states and walks the sequence one step
// at a time, keeping its states in registers from the first step to the last ("ufo.work"
// page, §1.1: h_t = exp(Delta_t A) h_{t-1} + Delta_t B_t u_t, y_t = C_t h_t; §3.2: channels
// are independent).  Nothing has to be composed across lanes: the state entering every step
// is already known, so each exponential exp(Delta A) is evaluated once and used once, with
// no segment operators, no warp scan and no second pass.  The parallelism comes from the
// channels (and sequences) alone, so the host picks this kernel only when there are enough
// of them to fill the GPU; a single long sequence goes to the chunked kernel instead.
//
// Per step and lane: x = Delta A log2(e) and a = ex2(x) for NS states, b = (Delta u) B,
// h = a h + b and y += C h.  The arithmetic is packed f32x2 over pairs of consecutive steps of
// one state (x, b and the y update; the recurrence itself is a scalar chain per state), so no
// operand has to be duplicated into a register pair.  Delta = softplus(delta + bias) and
// Delta u are evaluated once per (step, channel) by the whole CTA when a chunk lands, into
// shared memory, where the LPC lanes of a channel read them; after every block of 8 steps the
// LPC partial sums of y are reduced by recursive halving so that lane g ends with the full y
// of steps [g SUB, (g + 1) SUB) (SUB = 8 / LPC), which it gates (silu(z), skip term D u) and
// stores.
//
// Staging.  A CTA (four warps, CT channels of one sequence) copies the u, delta, z rows of
// its channels and the B, C rows of a TC-step chunk into shared memory with TMA bulk copies
// (cp.async.bulk completing on an mbarrier, no multicast), double-buffered: chunk c + 1
// streams in while chunk c is computed.  When a chunk has landed the CTA widens B and C to
// float32 (rows padded by 16 bytes so that the rows of a load phase hit distinct banks) and
// evaluates Delta and Delta u into double-buffered float32 rows; a lane then reads four steps
// of a state's B or C, or of its channel's Delta, with one 16-byte load that the other
// channels' lanes share (broadcast).
//
// Scheduling.  Work units are (sequence, channel tile) pairs taken from an atomic ticket by
// a persistent grid.  Packed sequences are visited longest first (ranked in every CTA from
// cu_seqlens), so that long units start early and short ones fill the tail.
//
// Windows start at the sequence start rounded down to a 16-byte boundary; steps outside
// [seq_start, seq_end) are identities (Delta = 0, Delta u = 0, b = 0) and are not stored,
// which also restarts the state at every packed-sequence boundary ("ufo.work" §4.2).
#pragma once

#include "common.cuh"

namespace ssm {

template <typename T, int N, int LPC, int TC, int W>
struct SeqCfg {
  static constexpr int kNS = N / LPC;       // states per lane
  static constexpr int kCPW = 32 / LPC;     // channels per warp
  static constexpr int kWarps = W;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kCT = kWarps * kCPW;  // channels per CTA
  static constexpr int kSub = 8 / LPC;      // steps of an 8-step block that a lane finishes
  // u/delta/z row pitch (elements): one 8-step block of padding, so that the channels of a
  // load phase hit distinct banks
  static constexpr int kXP = TC + 8;
  static constexpr size_t kXElems = size_t(3) * kCT * kXP;  // one staging buffer: u, delta, z
  static constexpr size_t kBCElems = size_t(2) * N * TC;    // one staging buffer: B, C
  // widened float32 rows (B then C, 2N rows of pitch kBP) and Delta, Delta u rows ([2][CT][kBP]):
  // 16 bytes of padding per row, and each group of NS state rows (the rows one lane reads)
  // shifted by 16 bytes more, so that the LPC lanes of a channel read distinct banks
  static constexpr int kBP = TC + 4;
  static constexpr size_t kBFElems = size_t(2) * N * kBP + 2 * LPC * 4;
  __host__ __device__ static constexpr int bf_row(int r) { return r * kBP + (r / kNS) * 4; }
  static constexpr size_t kDLElems = size_t(2) * kCT * kBP;
  static constexpr size_t kSmemBytes = 2 * kXElems * sizeof(T) + 2 * kBCElems * sizeof(T) +
                                       2 * (kBFElems + kDLElems) * sizeof(float) + kMaxSortedSeqs * sizeof(int);
  static_assert(N % LPC == 0 && kNS % 2 == 0, "whole pairs of states per lane");
  static_assert(8 % LPC == 0 && TC % 8 == 0, "8-step blocks");
  static_assert((kXP * sizeof(T)) % 16 == 0 && (TC * sizeof(T)) % 16 == 0, "16-byte rows");
  static_assert(((size_t(2) * kXElems + 2 * kBCElems) * sizeof(T)) % 16 == 0, "aligned float buffers");
};

// SUB consecutive elements of a staged row -> float32 (SUB * sizeof(T) bytes, aligned to it).
template <typename T, int SUB> __device__ __forceinline__ void load_sub(const T *p, float *f) {
  constexpr int kBytes = SUB * int(sizeof(T));
  if constexpr (kBytes == 32) {
    unpack16<T>(reinterpret_cast<const uint4 *>(p)[0], f);
    unpack16<T>(reinterpret_cast<const uint4 *>(p)[1], f + 16 / sizeof(T));
  } else if constexpr (kBytes == 16) {
    unpack16<T>(*reinterpret_cast<const uint4 *>(p), f);
  } else if constexpr (std::is_same<T, float>::value) {
#pragma unroll
    for (int j = 0; j < SUB; ++j) f[j] = p[j];
  } else if constexpr (kBytes == 8) {
    const uint2 v = *reinterpret_cast<const uint2 *>(p);
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
  } else {
    static_assert(kBytes == 4, "sub-vector size");
    const uint32_t v = *reinterpret_cast<const uint32_t *>(p);
    f[0] = __uint_as_float(v << 16); f[1] = __uint_as_float(v & 0xffff0000u);
  }
}

// SUB float32 values -> SUB consecutive output elements (aligned to SUB * sizeof(TO)).
template <typename TO, int SUB> __device__ __forceinline__ void store_sub(TO *p, const float *f) {
  if constexpr (std::is_same<TO, float>::value) {
    if constexpr (SUB % 4 == 0) {
#pragma unroll
      for (int v = 0; v < SUB / 4; ++v)
        reinterpret_cast<float4 *>(p)[v] = make_float4(f[4 * v], f[4 * v + 1], f[4 * v + 2], f[4 * v + 3]);
    } else if constexpr (SUB == 2) {
      *reinterpret_cast<float2 *>(p) = make_float2(f[0], f[1]);
    } else {
      p[0] = f[0];
    }
  } else {
    if constexpr (SUB == 8) {
      *reinterpret_cast<uint4 *>(p) = pack16<TO>(f);
    } else if constexpr (SUB == 4) {
      *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
    } else if constexpr (SUB == 2) {
      *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(f[0], f[1]);
    } else {
      p[0] = Elem<TO>::from_f32(f[0]);
    }
  }
}

template <typename T, typename TO, int N, int LPC, int TC, int W, bool HAS_Z>
__global__ void __launch_bounds__(W * 32, (LPC == 1 ? 8 : 16) / W) seq_scan_kernel(const ScanArgs args) {
  using Cfg = SeqCfg<T, N, LPC, TC, W>;
  constexpr int NS = Cfg::kNS, CPW = Cfg::kCPW, CT = Cfg::kCT, NT = Cfg::kThreads, XP = Cfg::kXP;
  constexpr int SUB = Cfg::kSub;
  constexpr int V = Elem<T>::kVec;
  constexpr bool kFast = Elem<T>::kFast;
  constexpr int nx = HAS_Z ? 3 : 2;

  extern __shared__ __align__(16) unsigned char smem[];
  T *const xs0 = reinterpret_cast<T *>(smem);           // [2][3][CT][XP]
  T *const bcs0 = xs0 + 2 * Cfg::kXElems;               // [2][2][N][TC]
  float *const bf0 = reinterpret_cast<float *>(bcs0 + 2 * Cfg::kBCElems);  // [2][2N][BP]
  float *const dl0 = bf0 + 2 * Cfg::kBFElems;                               // [2][2][CT][BP]
  int *const order = reinterpret_cast<int *>(dl0 + 2 * Cfg::kDLElems);      // [kMaxSortedSeqs]
  constexpr int BP = Cfg::kBP;
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int unit_sh;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int g = lane % LPC;                  // state group: states [g NS, (g + 1) NS)
  const int ch = warp * CPW + lane / LPC;    // channel within the tile
  const int64_t seqlen_r = (args.seqlen + V - 1) / V * V;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init_fence();
  }
  // rank packed sequences by length (descending, ties by index); order[rank] = sequence
  const bool sorted = args.cu_seqlens != nullptr && args.nseq <= kMaxSortedSeqs;
  if (sorted) {
    for (int i = threadIdx.x; i < args.nseq; i += NT) {
      const int li = args.cu_seqlens[i + 1] - args.cu_seqlens[i];
      int rank = 0;
      for (int j = 0; j < args.nseq; ++j) {
        const int lj = args.cu_seqlens[j + 1] - args.cu_seqlens[j];
        rank += (lj > li) || (lj == li && j < i);
      }
      order[rank] = i;
    }
  }
  __syncthreads();
  uint32_t gc = 0;  // chunks staged by this CTA so far: selects buffer and barrier parity

  for (;;) {
    if (threadIdx.x == 0) unit_sh = int(atomicAdd(args.ticket, 1u));
    __syncthreads();
    const int unit = unit_sh;
    if (unit >= args.total_units) break;
    const int tile = unit % args.ntiles;
    int s = unit / args.ntiles;
    if (sorted) s = order[s];
    const int grp = tile / args.tiles_per_group;
    const int64_t d0 = int64_t(grp) * args.group_dim + int64_t(tile % args.tiles_per_group) * CT;
    const int64_t d_end = min64(int64_t(grp + 1) * args.group_dim, args.dim);
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
    bcbase += int64_t(grp) * args.bc_group_stride;
    const int64_t w0 = t_lo & ~int64_t(V - 1);
    const int nchunks = t_hi > t_lo ? int((t_hi - w0 + TC - 1) / TC) : 0;
    const int nvalid = int(min64(CT, d_end - d0));
    const int64_t d = d0 + ch;
    const bool ch_ok = d < d_end;
    int64_t srow = s;  // row of this sequence's state in h0 / h_last; -1: bad pool slot
    if (args.state_slots) {
      srow = args.state_slots[s];
      if (srow < 0 || srow >= args.num_slots) {
        if (threadIdx.x == 0 && tile == 0) report_status(4 /* SSM_ERR_BAD_SLOT */);
        srow = -1;
      }
    }

    // per-lane constants and the state entering the sequence
    // per-lane constants (A log2(e) of each state, duplicated for step-pair arithmetic) and the
    // state entering the sequence
    float2 A2[NS];
    float h[NS];
    float Dd = 0.f;
    [[maybe_unused]] float bias = 0.f;
#pragma unroll
    for (int n = 0; n < NS; ++n) {
      A2[n] = make_float2(0.f, 0.f);
      h[n] = 0.f;
    }
    if (ch_ok) {
      const float *Ar = args.A + d * N + g * NS;
#pragma unroll
      for (int n = 0; n < NS; ++n) A2[n] = make_float2(Ar[n] * kLog2e, Ar[n] * kLog2e);
      if (args.h0 && srow >= 0) {
        const float *hr = args.h0 + (srow * args.dim + d) * N + g * NS;
#pragma unroll
        for (int n = 0; n < NS; ++n) h[n] = hr[n];
      }
      Dd = args.Dskip ? args.Dskip[d] : 0.f;
      bias = args.bias ? args.bias[d] : 0.f;
    }

    // TMA: chunk c's u/delta/z rows of the tile and B/C rows into buffer `buf`
    auto issue_chunk = [&](int buf, int c) {
      const int64_t wstart = w0 + int64_t(c) * TC;
      const int64_t wend = min64(wstart + TC, seqlen_r);
      const uint32_t row_bytes = uint32_t((wend - wstart) * int64_t(sizeof(T)));
      T *xd = xs0 + buf * Cfg::kXElems;
      T *bd = bcs0 + buf * Cfg::kBCElems;
      fence_proxy_async_smem();
      if (threadIdx.x == 0) mbar_arrive_expect_tx(&bars[buf], row_bytes * uint32_t(nx * nvalid + 2 * N));
      for (int r = threadIdx.x; r < nx * CT + 2 * N; r += NT) {
        if (r < nx * CT) {
          const int which = r / CT, c2 = r % CT;
          if (c2 >= nvalid) continue;
          const T *base = static_cast<const T *>(which == 0 ? args.u : (which == 1 ? args.delta : args.z));
          bulk_g2s(xd + size_t(r) * XP, base + xbase + (d0 + c2) * args.x_dim_stride + wstart, row_bytes,
                   &bars[buf]);
        } else {
          const int r2 = r - nx * CT, which = r2 / N, n = r2 % N;
          const T *base = static_cast<const T *>(which == 0 ? args.B : args.C);
          bulk_g2s(bd + size_t(r2) * TC, base + bcbase + int64_t(n) * args.bc_state_stride + wstart, row_bytes,
                   &bars[buf]);
        }
      }
    };

    // One chunk of this lane's steps; the masked instance handles chunks that straddle a
    // sequence boundary or the end of the rows (Delta and Delta u are already zero there).
    auto compute_chunk = [&](auto masked_tag, const T *X, const float *Bf, const float *Dl, int64_t wstart,
                             int rel_lo, int rel_hi) {
      constexpr bool kMasked = decltype(masked_tag)::value;
      [[maybe_unused]] const T *ru = X + size_t(ch) * XP;
      [[maybe_unused]] const T *rz = X + size_t(2 * CT + ch) * XP;
      const float *Bb = Bf + Cfg::bf_row(g * NS);       // rows of this lane's states
      const float *Cb = Bf + Cfg::bf_row(N + g * NS);
      const float *rdl = Dl + size_t(ch) * BP;           // Delta of this channel
      const float *rdu = Dl + size_t(CT + ch) * BP;      // Delta u
#pragma unroll 1
      for (int blk = 0; blk < TC / 8; ++blk) {
        float dl[8], dU[8];
        if constexpr (LPC == 1) {
          // the lane owns its channel: Delta and Delta u of the block's 8 steps, here
          float uv[8], dv[8];
          load_sub<T, 8>(ru + blk * 8, uv);
          load_sub<T, 8>(X + size_t(CT + ch) * XP + blk * 8, dv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float dt = softplus_t<kFast>(dv[j] + bias);
            if constexpr (kMasked) {
              const bool in = blk * 8 + j >= rel_lo && blk * 8 + j < rel_hi;
              dl[j] = in ? dt : 0.f;
              dU[j] = in ? dt * uv[j] : 0.f;  // select: a non-finite u outside the sequence stays out
            } else {
              dl[j] = dt;
              dU[j] = dt * uv[j];
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float4 l4 = reinterpret_cast<const float4 *>(rdl + blk * 8)[q];
            const float4 u4 = reinterpret_cast<const float4 *>(rdu + blk * 8)[q];
            dl[4 * q] = l4.x; dl[4 * q + 1] = l4.y; dl[4 * q + 2] = l4.z; dl[4 * q + 3] = l4.w;
            dU[4 * q] = u4.x; dU[4 * q + 1] = u4.y; dU[4 * q + 2] = u4.z; dU[4 * q + 3] = u4.w;
          }
        }
        // ---- the recurrence over the block's 8 steps for this lane's NS states, in step pairs
        float2 yp2[4];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) yp2[k2] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
#pragma unroll
          for (int n = 0; n < NS; ++n) {
            const float4 b4 = reinterpret_cast<const float4 *>(Bb + size_t(n) * BP + blk * 8)[q];
            const float4 c4 = reinterpret_cast<const float4 *>(Cb + size_t(n) * BP + blk * 8)[q];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int k2 = 2 * q + e;
              const float2 dd = make_float2(dl[2 * k2], dl[2 * k2 + 1]);
              const float2 uu = make_float2(dU[2 * k2], dU[2 * k2 + 1]);
              const float2 x = __fmul2_rn(dd, A2[n]);
              const float2 a = make_float2(ex2_approx(x.x), ex2_approx(x.y));
              float2 bb = __fmul2_rn(uu, e ? make_float2(b4.z, b4.w) : make_float2(b4.x, b4.y));
              if constexpr (kMasked) {
                // stale B outside the sequence never reaches h (Delta u is 0 there, B may be non-finite)
                bb.x = uu.x != 0.f ? bb.x : 0.f;
                bb.y = uu.y != 0.f ? bb.y : 0.f;
              }
              const float h0v = fmaf(a.x, h[n], bb.x);
              h[n] = fmaf(a.y, h0v, bb.y);
              yp2[k2] = __ffma2_rn(e ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y), make_float2(h0v, h[n]),
                                     yp2[k2]);
            }
          }
        }
        float yp[8];
#pragma unroll
        for (int k2 = 0; k2 < 4; ++k2) {
          yp[2 * k2] = yp2[k2].x;
          yp[2 * k2 + 1] = yp2[k2].y;
        }
        // ---- sum y over the channel's LPC lanes by recursive halving: at each level a lane
        // keeps the half of its step range picked by one bit of g and sends the other half to
        // the partner lane; lane g ends with steps [g SUB, (g + 1) SUB)
#pragma unroll
        for (int lev = 0; (1 << lev) < LPC; ++lev) {
          const int off = LPC >> (lev + 1);
          const int half = 8 >> (lev + 1);
          const bool upper = (g & off) != 0;
#pragma unroll
          for (int j = 0; j < half; ++j) {
            const float send = upper ? yp[j] : yp[half + j];
            const float keep = upper ? yp[half + j] : yp[j];
            yp[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
          }
        }
        // ---- skip term, gate, store this lane's SUB steps
        if (ch_ok) {
          const int c0 = blk * 8 + g * SUB;
          float uv[SUB], o[SUB];
          [[maybe_unused]] float zv[SUB];
          load_sub<T, SUB>(ru + c0, uv);
          if constexpr (HAS_Z) load_sub<T, SUB>(rz + c0, zv);
#pragma unroll
          for (int j = 0; j < SUB; ++j) {
            float v = fmaf(Dd, uv[j], yp[j]);
            if constexpr (HAS_Z) v *= silu_t<kFast>(zv[j]);
            o[j] = v;
          }
          TO *gy = static_cast<TO *>(args.y) + xbase + d * args.x_dim_stride + wstart + c0;
          if (!kMasked || (c0 >= rel_lo && c0 + SUB <= rel_hi)) {
            store_sub<TO, SUB>(gy, o);
          } else {
#pragma unroll
            for (int j = 0; j < SUB; ++j)
              if (c0 + j >= rel_lo && c0 + j < rel_hi) gy[j] = Elem<TO>::from_f32(o[j]);
          }
        }
      }
    };

    // ------------------------------------------------------------- the unit's chunks
    if (nchunks > 0) issue_chunk(int(gc & 1u), 0);
    for (int c = 0; c < nchunks; ++c, ++gc) {
      const int buf = int(gc & 1u);
      const int64_t wstart = w0 + int64_t(c) * TC;
      const bool landed = mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);
      const int rel_lo = int(max64(t_lo - wstart, -1));
      const int rel_hi = int(min64(t_hi - wstart, TC + 1));
      {
        // widen the chunk's B and C to float32 rows
        const T *bs = bcs0 + buf * Cfg::kBCElems;
        float *bf = bf0 + buf * Cfg::kBFElems;
        for (int i = threadIdx.x; i < 2 * N * (TC / 8); i += NT) {
          const int row = i % (2 * N), blk = i / (2 * N);
          float f[8];
          load_sub<T, 8>(bs + size_t(row) * TC + blk * 8, f);
          float4 *dst = reinterpret_cast<float4 *>(bf + Cfg::bf_row(row) + blk * 8);
          dst[0] = make_float4(f[0], f[1], f[2], f[3]);
          dst[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
        // Delta = softplus(delta + bias) and Delta u, once per (step, channel), for the LPC
        // lanes of a channel to share; steps outside the sequence are identities (Delta =
        // Delta u = 0).  With LPC = 1 the lane evaluates its own.
        const T *Xs = xs0 + buf * Cfg::kXElems;
        float *dlw = dl0 + buf * Cfg::kDLElems;
        for (int i = threadIdx.x; i < (LPC > 1 ? CT * (TC / 8) : 0); i += NT) {
          const int c2 = i % CT, blk = i / CT;
          const int64_t dd = d0 + c2;
          const float bias = (dd < d_end && args.bias) ? args.bias[dd] : 0.f;
          float uv[8], dv[8], o1[8], o2[8];
          load_sub<T, 8>(Xs + size_t(c2) * XP + blk * 8, uv);
          load_sub<T, 8>(Xs + size_t(CT + c2) * XP + blk * 8, dv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int t = blk * 8 + j;
            const bool in = t >= rel_lo && t < rel_hi;
            const float dt = softplus_t<kFast>(dv[j] + bias);
            o1[j] = in ? dt : 0.f;
            o2[j] = in ? dt * uv[j] : 0.f;  // select: a non-finite u outside the sequence stays out
          }
          float4 *w1 = reinterpret_cast<float4 *>(dlw + size_t(c2) * BP + blk * 8);
          float4 *w2 = reinterpret_cast<float4 *>(dlw + size_t(CT + c2) * BP + blk * 8);
          w1[0] = make_float4(o1[0], o1[1], o1[2], o1[3]);
          w1[1] = make_float4(o1[4], o1[5], o1[6], o1[7]);
          w2[0] = make_float4(o2[0], o2[1], o2[2], o2[3]);
          w2[1] = make_float4(o2[4], o2[5], o2[6], o2[7]);
        }
      }
      // chunk c widened; every warp is done with chunk c-1's buffers
      if (__syncthreads_or(!landed)) {
        // a copy did not land within the bounded wait (SSM_ERR_TIMEOUT is recorded): give up
        // on this CTA's work, once more waiting (bounded) for the copy in flight so that it
        // does not write shared memory after the CTA has exited
        mbar_wait_bounded(&bars[buf], (gc >> 1) & 1u);
        return;
      }
      if (c + 1 < nchunks) issue_chunk(buf ^ 1, c + 1);  // streams in while chunk c is computed
      const T *X = xs0 + buf * Cfg::kXElems;
      const float *Bf = bf0 + buf * Cfg::kBFElems;
      const float *Dl = dl0 + buf * Cfg::kDLElems;
      if (rel_lo <= 0 && rel_hi >= TC)
        compute_chunk(std::false_type{}, X, Bf, Dl, wstart, rel_lo, rel_hi);
      else
        compute_chunk(std::true_type{}, X, Bf, Dl, wstart, rel_lo, rel_hi);
    }

    // ------------------------------------------------------------- final state
    if (args.h_last && srow >= 0 && ch_ok) {
      float *hr = args.h_last + (srow * args.dim + d) * N + g * NS;
#pragma unroll
      for (int n = 0; n < NS; ++n) hr[n] = h[n];
    }
    __syncthreads();  // shared state of this unit is dead before the next unit overwrites it
  }
}

}  // namespace ssm
