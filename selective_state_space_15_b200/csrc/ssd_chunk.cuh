// SSD (state-space duality) chunked form of the scan on the sm_100a tensor cores.
//
// The second article of the "会议长序列建模…" page (ufo.work), "Mamba-2/SSD架构下的矩阵化加速范式…",
// §1.1 and §2.2: with a scalar decay A_h per head and a step Delta_t shared by the head's P
// channels, the scan over one chunk of T steps is a masked matrix product,
//
//   cum_t   = sum_{k <= t} Delta_k A_h                      (prefix sum inside the chunk)
//   S[t][s] = (C_t . B_s) exp(cum_t - cum_s)  for s <= t, 0 otherwise
//   Y[t][p] = sum_s S[t][s] V[s][p] + exp(cum_t) sum_n C_t[n] H[p][n],   V[s][p] = x[p][s] Delta_s
//   H'[n][p] = exp(cum_T) H[n][p] + sum_s B_s[n] exp(cum_T - cum_s) V[s][p]
//
// with the state H [P][N] carried from chunk to chunk (the chunk-boundary states of its §3.1).
// All four products are dense and go to tcgen05.mma (kind::f16, float16 operands in shared
// memory, float32 accumulators in tensor memory):
//   G  = C^T B^T:  [T=128 t][T=128 s] over K = N (the states),
//   Y  = M V^T + C'^T H^T: [128 t][P] over K = T, then K = N (M = G masked and decayed, C' = C
//        scaled per t by exp(cum_t)),
//   H' = B V'^T accumulated onto exp(cum_T) H: [N=128 n][P] over K = T (V' = V scaled per s by
//        exp(cum_T - cum_s)).
// The mask, the decays and the state rescaling are applied by the CUDA cores between the
// products (each thread owns one row: t for G and Y, n for the state).  float16 keeps 11
// significant bits: the bf16 inputs are represented exactly, the computed operands (M, V, V',
// C', H) are rounded once, and every sum is accumulated in float32.
//
// One CTA (four warps, 128 threads) per (sequence, head) walks the chunks in order.  Shared
// memory: seven operand tiles (176 KB); tensor memory: 256 columns (G, Y, the state).
#pragma once

#include "common.cuh"
#include "tcgen05.cuh"

namespace ssm {

struct SsdArgs {
  const __nv_bfloat16 *x;  // [batch][H][P][L]
  const float *dt;         // [batch][H][L]
  const float *A;          // [H]
  const __nv_bfloat16 *B;  // [batch][N][L]
  const __nv_bfloat16 *C;  // [batch][N][L]
  const float *h0;         // [batch][H][P][N] or nullptr
  __nv_bfloat16 *y;        // [batch][H][P][L]
  float *h_last;           // [batch][H][P][N] or nullptr
  int64_t nheads, seqlen;
};

constexpr int kSsdT = 128;   // chunk length
constexpr int kSsdP = 64;    // head dimension
constexpr int kSsdN = 128;   // state size
constexpr uint32_t kSsdTmemCols = 256;
// shared-memory tiles (bytes); each 128 x 128 operand is two 128-row tiles of 64 K-elements
constexpr uint32_t kSsdTile128 = 128 * 128 * 2;  // 32 KB
constexpr uint32_t kSsdTile64 = 64 * 128 * 2;    // 16 KB
constexpr uint32_t kSsdOffCT = 0;                       // C^T then C'^T [t][n]
constexpr uint32_t kSsdOffBT = kSsdOffCT + kSsdTile128;  // B^T [s][n]
constexpr uint32_t kSsdOffBN = kSsdOffBT + kSsdTile128;  // B [n][s]
constexpr uint32_t kSsdOffM = kSsdOffBN + kSsdTile128;   // M [t][s]
constexpr uint32_t kSsdOffV = kSsdOffM + kSsdTile128;    // V [p][s]
constexpr uint32_t kSsdOffVS = kSsdOffV + kSsdTile64;    // V' [p][s]
constexpr uint32_t kSsdOffH = kSsdOffVS + kSsdTile64;    // H [p][n]
constexpr uint32_t kSsdOffCum = kSsdOffH + kSsdTile64;   // cum [128] float
constexpr uint32_t kSsdSmemBytes = kSsdOffCum + kSsdT * 4 + 1024;  // + slack to align the base to 1024

// Write 8 float16 values (K-elements 8j .. 8j+7 of row r) into a K-major swizzled operand
// whose K extent is split into 64-element tiles of `rows` rows each.
__device__ __forceinline__ void ssd_put8(unsigned char *tile, uint32_t rows, uint32_t r, uint32_t k0,
                                         const float (&v)[8]) {
  const uint32_t kb = k0 >> 6, kk = k0 & 63u;
  __half2 h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4 *>(tile + kb * rows * 128u + tc::sw128_offset(r, kk)) = *reinterpret_cast<uint4 *>(h);
}

__global__ void __launch_bounds__(128, 1) ssd_chunk_kernel(const SsdArgs args) {
  constexpr int T = kSsdT, P = kSsdP, N = kSsdN;
  extern __shared__ unsigned char ssd_smem_raw[];
  // operand tiles start on a 1024-byte boundary (the swizzle atom)
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(ssd_smem_raw) + 1023) & ~uintptr_t(1023));
  float *cum = reinterpret_cast<float *>(smem + kSsdOffCum);
  __shared__ __align__(8) uint64_t bar_g, bar_y;
  __shared__ uint32_t tmem_slot;
  __shared__ float warp_sum[4];

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int64_t bh = blockIdx.x;                 // (sequence, head)
  const int64_t b = bh / args.nheads, h = bh % args.nheads;
  const int64_t L = args.seqlen;
  const float Ah = args.A[h];
  const __nv_bfloat16 *xg = args.x + bh * P * L;
  const float *dtg = args.dt + bh * L;
  const __nv_bfloat16 *Bg = args.B + b * N * L;
  const __nv_bfloat16 *Cg = args.C + b * N * L;

  if (warp == 0) {
    tc::tmem_alloc(&tmem_slot, kSsdTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_g, 1);
    mbar_init(&bar_y, 1);
    mbar_init_fence();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = tmem_slot;
  const uint32_t t_G = tmem, t_Y = tmem + 128, t_H = tmem + 192;      // column bases
  const uint32_t lane_base = uint32_t(warp * 32) << 16;               // this warp's lanes

  // the state: tensor memory [n][p] (thread n owns lane n), float32; h0 or zero
  {
    float v[16];
#pragma unroll
    for (int c = 0; c < P / 16; ++c) {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = args.h0 ? args.h0[(bh * P + c * 16 + i) * N + tid] : 0.f;
      tc::tmem_st16(t_H + lane_base + c * 16, v);
    }
    tc::tmem_wait_st();
  }

  const uint32_t idesc_tt = tc::idesc_f16_f32(128, 128);  // G: M = 128 (t), N = 128 (s)
  const uint32_t idesc_tp = tc::idesc_f16_f32(128, P);    // Y and the state: N = P = 64
  const uint32_t a_CT = tc::smem_addr(smem + kSsdOffCT), a_BT = tc::smem_addr(smem + kSsdOffBT);
  const uint32_t a_BN = tc::smem_addr(smem + kSsdOffBN), a_M = tc::smem_addr(smem + kSsdOffM);
  const uint32_t a_V = tc::smem_addr(smem + kSsdOffV), a_VS = tc::smem_addr(smem + kSsdOffVS);
  const uint32_t a_H = tc::smem_addr(smem + kSsdOffH);
  const int nchunks = int((L + T - 1) / T);

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = int64_t(c) * T;
    const int64_t tt = t0 + tid;                // this thread's step (row t of G and Y)
    const bool t_ok = tt < L;
    // ---- prefix sum of Delta A over the chunk (steps past the end add 0)
    float v = t_ok ? dtg[tt] * Ah : 0.f;
#pragma unroll
    for (int off = 1; off < 32; off *= 2) {
      const float o = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += o;
    }
    if (lane == 31) warp_sum[warp] = v;
    __syncthreads();
    for (int w = 0; w < warp; ++w) v += warp_sum[w];
    cum[tid] = v;
    __syncthreads();
    const float cum_t = v, cum_T = cum[T - 1];

    // ---- operand tiles (thread tid: row t of C^T and B^T, row n of B, row p of V / V')
    {
      float cv[8], bv[8];
#pragma unroll 1
      for (int n0 = 0; n0 < N; n0 += 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          cv[i] = t_ok ? __bfloat162float(Cg[(n0 + i) * L + tt]) : 0.f;
          bv[i] = t_ok ? __bfloat162float(Bg[(n0 + i) * L + tt]) : 0.f;
        }
        ssd_put8(smem + kSsdOffCT, 128, tid, n0, cv);
        ssd_put8(smem + kSsdOffBT, 128, tid, n0, bv);
      }
      // B [n][s]: row n = tid, 16-byte loads along the sequence
      const __nv_bfloat16 *brow = Bg + int64_t(tid) * L + t0;
#pragma unroll 1
      for (int s0 = 0; s0 < T; s0 += 8) {
        float f[8];
        if (t0 + s0 + 8 <= L) {
          unpack16<__nv_bfloat16>(*reinterpret_cast<const uint4 *>(brow + s0), f);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = t0 + s0 + i < L ? __bfloat162float(brow[s0 + i]) : 0.f;
        }
        ssd_put8(smem + kSsdOffBN, 128, tid, s0, f);
      }
      // V [p][s] = x[p][s] Delta_s and V' = V exp(cum_T - cum_s): two threads per row p
      const int p = tid >> 1, half = tid & 1;
      const __nv_bfloat16 *xrow = xg + int64_t(p) * L + t0;
#pragma unroll 1
      for (int s0 = half * 64; s0 < half * 64 + 64; s0 += 8) {
        float f[8], fv[8], fs[8];
        if (t0 + s0 + 8 <= L) {
          unpack16<__nv_bfloat16>(*reinterpret_cast<const uint4 *>(xrow + s0), f);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = t0 + s0 + i < L ? __bfloat162float(xrow[s0 + i]) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int64_t ts = t0 + s0 + i;
          const float d = ts < L ? dtg[ts] : 0.f;
          fv[i] = f[i] * d;
          fs[i] = fv[i] * __expf(cum_T - cum[s0 + i]);
        }
        ssd_put8(smem + kSsdOffV, 64, p, s0, fv);
        ssd_put8(smem + kSsdOffVS, 64, p, s0, fs);
      }
      // H [p][n] from the state (thread n reads its tensor-memory lane: the P values of row n)
      float hv[16];
#pragma unroll
      for (int cb = 0; cb < P / 16; ++cb) {
        tc::tmem_ld16(t_H + lane_base + cb * 16, hv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint32_t pp = cb * 16 + i, kb = uint32_t(tid) >> 6, kk = uint32_t(tid) & 63u;
          *reinterpret_cast<__half *>(smem + kSsdOffH + kb * 64u * 128u + tc::sw128_offset(pp, kk)) =
              __float2half_rn(hv[i]);
        }
      }
    }
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    // ---- G = C^T B^T (K = N: 2 tiles x 4 steps of 16)
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_f16(t_G, tc::sdesc_k_sw128(a_CT + kb * 128 * 128 + ks * 32),
                      tc::sdesc_k_sw128(a_BT + kb * 128 * 128 + ks * 32), idesc_tt, (kb | ks) != 0);
      tc::commit(&bar_g);
    }
    mbar_wait_bounded(&bar_g, uint32_t(c & 1));
    tc::fence_after_sync();

    // ---- M[t][s] = G exp(cum_t - cum_s) (s <= t), C' = C exp(cum_t), state *= exp(cum_T)
    {
#pragma unroll 1
      for (int s0 = 0; s0 < T; s0 += 16) {
        float g[16];
        tc::tmem_ld16(t_G + lane_base + s0, g);
        tc::tmem_wait_ld();
        float m0[8], m1[8];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int s = s0 + i;
          const float m = s <= tid ? g[i] * __expf(cum_t - cum[s]) : 0.f;
          if (i < 8) m0[i] = m; else m1[i - 8] = m;
        }
        ssd_put8(smem + kSsdOffM, 128, tid, s0, m0);
        ssd_put8(smem + kSsdOffM, 128, tid, s0 + 8, m1);
      }
      const float e_t = __expf(cum_t);
#pragma unroll 1
      for (int n0 = 0; n0 < N; n0 += 8) {
        const uint32_t kb = uint32_t(n0) >> 6;
        unsigned char *q = smem + kSsdOffCT + kb * 128u * 128u + tc::sw128_offset(tid, n0 & 63);
        __half2 *hq = reinterpret_cast<__half2 *>(q);
#pragma unroll
        for (int i = 0; i < 4; ++i) hq[i] = __hmul2(hq[i], __float2half2_rn(e_t));
      }
      const float e_T = __expf(cum_T);
      float hv[16];
#pragma unroll
      for (int cb = 0; cb < P / 16; ++cb) {
        tc::tmem_ld16(t_H + lane_base + cb * 16, hv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) hv[i] *= e_T;
        tc::tmem_st16(t_H + lane_base + cb * 16, hv);
      }
      tc::tmem_wait_st();
    }
    tc::fence_async_smem();
    tc::fence_before_sync();
    __syncthreads();

    // ---- Y = M V^T + C'^T H^T; state += B V'^T
    if (tid == 0) {
      tc::fence_after_sync();
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_f16(t_Y, tc::sdesc_k_sw128(a_M + kb * 128 * 128 + ks * 32),
                      tc::sdesc_k_sw128(a_V + kb * 64 * 128 + ks * 32), idesc_tp, (kb | ks) != 0);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_f16(t_Y, tc::sdesc_k_sw128(a_CT + kb * 128 * 128 + ks * 32),
                      tc::sdesc_k_sw128(a_H + kb * 64 * 128 + ks * 32), idesc_tp, 1u);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_f16(t_H, tc::sdesc_k_sw128(a_BN + kb * 128 * 128 + ks * 32),
                      tc::sdesc_k_sw128(a_VS + kb * 64 * 128 + ks * 32), idesc_tp, 1u);
      tc::commit(&bar_y);
    }
    mbar_wait_bounded(&bar_y, uint32_t(c & 1));
    tc::fence_after_sync();

    // ---- y[p][t] for this thread's step; the final state
    {
      float yv[16];
#pragma unroll
      for (int cb = 0; cb < P / 16; ++cb) {
        tc::tmem_ld16(t_Y + lane_base + cb * 16, yv);
        tc::tmem_wait_ld();
        if (t_ok) {
#pragma unroll
          for (int i = 0; i < 16; ++i) args.y[(bh * P + cb * 16 + i) * L + tt] = __float2bfloat16_rn(yv[i]);
        }
      }
      if (c == nchunks - 1 && args.h_last) {
        float hv[16];
#pragma unroll
        for (int cb = 0; cb < P / 16; ++cb) {
          tc::tmem_ld16(t_H + lane_base + cb * 16, hv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) args.h_last[(bh * P + cb * 16 + i) * N + tid] = hv[i];
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
  }
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tmem, kSsdTmemCols);
}

}  // namespace ssm
