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
// One CTA (eight warps: two threads per row of every tile) per (sequence, head) walks the
// chunks in order.  Inputs are read with 16-byte loads along the time axis; the transposed
// operands (C^T, B^T: rows t) are formed in shared memory from the row-major copies (rows n).
// Shared memory: seven operand tiles (176 KB); tensor memory: 256 columns (G, Y, the state).
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
constexpr uint32_t kSsdOffCum = kSsdOffH + kSsdTile64;   // cum, dt, decay to the chunk end: 3 x [128] float
constexpr uint32_t kSsdSmemBytes = kSsdOffCum + 3 * kSsdT * 4 + 1024;  // + slack to align the base to 1024
constexpr int kSsdThreads = 256;

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

// 8 float32 values as float16 at byte `off` of a tile (a 16-byte chunk of a swizzled row).
__device__ __forceinline__ void ssd_st8(unsigned char *p, const float (&v)[8]) {
  __half2 h[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(v[2 * i], v[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = *reinterpret_cast<uint4 *>(h);
}
// 8 consecutive bf16 values of a row as they are stored (zeros past the sequence end).
__device__ __forceinline__ uint4 ssd_raw8(const __nv_bfloat16 *row, int64_t t, int64_t L) {
  if (t + 8 <= L) return *reinterpret_cast<const uint4 *>(row);
  uint16_t e[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) e[i] = t + i < L ? reinterpret_cast<const uint16_t *>(row)[i] : uint16_t(0);
  return make_uint4(e[0] | (uint32_t(e[1]) << 16), e[2] | (uint32_t(e[3]) << 16), e[4] | (uint32_t(e[5]) << 16),
                    e[6] | (uint32_t(e[7]) << 16));
}

__global__ void __launch_bounds__(kSsdThreads, 1) ssd_chunk_kernel(const SsdArgs args) {
  constexpr int T = kSsdT, P = kSsdP, N = kSsdN;
  extern __shared__ unsigned char ssd_smem_raw[];
  // operand tiles start on a 1024-byte boundary (the swizzle atom)
  unsigned char *smem = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(ssd_smem_raw) + 1023) & ~uintptr_t(1023));
  float *cum = reinterpret_cast<float *>(smem + kSsdOffCum);
  float *dts = cum + T;   // Delta of the chunk's steps (0 past the end)
  float *wdec = dts + T;  // exp(cum_T - cum_s): decay from step s to the chunk end
  unsigned char *tmp = smem + kSsdOffM;  // C [n][t] before the transpose; y [p][t] after the products
  __shared__ __align__(8) uint64_t bar_g, bar_y;
  __shared__ uint32_t tmem_slot;
  __shared__ float warp_sum[4];

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int r = tid & 127, hf = tid >> 7;           // tile row of this thread and its half of the row
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
  const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;         // this warp's lanes (= rows r)
  // Swizzled byte offsets (tc::sw128_offset) this thread uses every chunk: ro[j] = 16-byte chunk
  // j of row r (rows r of B, C, C^T, B^T, M); element (n, r) of a [n][K] tile with n = 8m + i
  // (column r read down the rows: the transposes, the H tile) lies at n * 128 + co[i].
  uint32_t ro[8], co[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ro[j] = tc::sw128_offset(uint32_t(r), uint32_t(8 * j));
    co[j] = tc::sw128_offset(uint32_t(j), uint32_t(r) & 63u) - uint32_t(j) * 128u;
  }
  const uint32_t rcol = (uint32_t(r) >> 6) * 128u * 128u;  // the 64-column tile of column r (128-row tiles)

  // the state: tensor memory [n][p] (lane n), float32; h0 or zero.  Thread (r, hf): lane r,
  // columns [32 hf, 32 hf + 32)
  {
    float v[16];
#pragma unroll
    for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = args.h0 ? args.h0[(bh * P + c * 16 + i) * N + r] : 0.f;
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

  // The raw inputs of a chunk, in registers: B and C rows n = r (half hf of the chunk's steps),
  // x row p = tid / 4 (a quarter), Delta of step r.  Loaded one chunk ahead, so that the global
  // loads of chunk c + 1 are in flight while chunk c is computed.
  uint4 rb[8], rc[8], rx[4];
  float rdt = 0.f;
  auto load_raw = [&](int cc) {
    const int64_t t0 = int64_t(cc) * T;
    const __nv_bfloat16 *brow = Bg + int64_t(r) * L + t0, *crow = Cg + int64_t(r) * L + t0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int s0 = hf * 64 + j * 8;
      rb[j] = ssd_raw8(brow + s0, t0 + s0, L);
      rc[j] = ssd_raw8(crow + s0, t0 + s0, L);
    }
    const int p = tid >> 2, q = tid & 3;
    const __nv_bfloat16 *xrow = xg + int64_t(p) * L + t0;
#pragma unroll
    for (int j = 0; j < 4; ++j) rx[j] = ssd_raw8(xrow + q * 32 + j * 8, t0 + q * 32 + j * 8, L);
    if (tid < T) rdt = t0 + r < L ? dtg[t0 + r] : 0.f;
  };
  load_raw(0);

  for (int c = 0; c < nchunks; ++c) {
    const int64_t t0 = int64_t(c) * T;
    // ---- Delta, the prefix sum of Delta A over the chunk (steps past the end add 0), decays
    if (tid < T) {
      const float dtv = rdt;
      dts[r] = dtv;
      float v = dtv * Ah;
#pragma unroll
      for (int off = 1; off < 32; off *= 2) {
        const float o = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += o;
      }
      if (lane == 31) warp_sum[warp] = v;
      cum[r] = v;  // the warp's part; the other warps' sums are added below
    }
    __syncthreads();
    if (tid < T) {
      float v = cum[r];
      for (int w = 0; w < warp; ++w) v += warp_sum[w];
      cum[r] = v;
    }
    __syncthreads();
    const float cum_t = cum[r], cum_T = cum[T - 1];
    if (tid < T) wdec[r] = __expf(cum_T - cum_t);

    // ---- B [n][s] and C [n][t] (row n = r, half hf of the chunk) from the registers
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float f[8];
      unpack16<__nv_bfloat16>(rb[j], f);
      ssd_st8(smem + kSsdOffBN + hf * 128 * 128 + ro[j], f);
      unpack16<__nv_bfloat16>(rc[j], f);
      ssd_st8(tmp + hf * 128 * 128 + ro[j], f);
    }
    __syncthreads();  // wdec, B and C in place
    // ---- V [p][s] = x[p][s] Delta_s and V' = V exp(cum_T - cum_s): four threads per row p
    {
      const int p = tid >> 2, q = tid & 3;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s0 = q * 32 + j * 8;
        float f[8], fs[8];
        unpack16<__nv_bfloat16>(rx[j], f);
        const float4 d0 = *reinterpret_cast<const float4 *>(dts + s0), d1 = *reinterpret_cast<const float4 *>(dts + s0 + 4);
        const float4 w0 = *reinterpret_cast<const float4 *>(wdec + s0), w1 = *reinterpret_cast<const float4 *>(wdec + s0 + 4);
        const float dd[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[i] *= dd[i];
          fs[i] = f[i] * ww[i];
        }
        ssd_put8(smem + kSsdOffV, 64, p, s0, f);
        ssd_put8(smem + kSsdOffVS, 64, p, s0, fs);
      }
    }
    if (c + 1 < nchunks) load_raw(c + 1);  // lands while this chunk is computed
    // ---- H [p][n] from the state (lane n = r holds row n; this thread's 32 columns p)
    {
      float hv[16];
#pragma unroll
      for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
        tc::tmem_ld16(t_H + lane_base + cb * 16, hv);
        tc::tmem_wait_ld();
        unsigned char *hcol = smem + kSsdOffH + (uint32_t(r) >> 6) * 64u * 128u + cb * 16 * 128;
#pragma unroll
        for (int i = 0; i < 16; ++i) *reinterpret_cast<__half *>(hcol + i * 128 + co[i & 7]) = __float2half_rn(hv[i]);
      }
    }
    // ---- C^T [t][n] and B^T [s][n] from the row-major copies (row t = r, states of half hf)
    {
      const unsigned char *ccol = tmp + rcol + hf * 64 * 128, *bcol = smem + kSsdOffBN + rcol + hf * 64 * 128;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        uint32_t cw[4], bw[4];
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          const uint32_t o0 = (8 * m + i) * 128 + co[i], o1 = (8 * m + i + 1) * 128 + co[i + 1];
          cw[i / 2] = *reinterpret_cast<const uint16_t *>(ccol + o0) |
                      (uint32_t(*reinterpret_cast<const uint16_t *>(ccol + o1)) << 16);
          bw[i / 2] = *reinterpret_cast<const uint16_t *>(bcol + o0) |
                      (uint32_t(*reinterpret_cast<const uint16_t *>(bcol + o1)) << 16);
        }
        *reinterpret_cast<uint4 *>(smem + kSsdOffCT + hf * 128 * 128 + ro[m]) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        *reinterpret_cast<uint4 *>(smem + kSsdOffBT + hf * 128 * 128 + ro[m]) = make_uint4(bw[0], bw[1], bw[2], bw[3]);
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
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int s0 = hf * 64 + 16 * m;
        float g[16];
        tc::tmem_ld16(t_G + lane_base + s0, g);
        tc::tmem_wait_ld();
        float m0[8], m1[8];
        if (s0 > r) {  // the block lies above the diagonal (s > t)
#pragma unroll
          for (int i = 0; i < 8; ++i) m0[i] = m1[i] = 0.f;
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float4 c4 = *reinterpret_cast<const float4 *>(cum + s0 + 4 * q);
            const float cs[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 4 * q + e;
              const float v = s0 + i <= r ? g[i] * __expf(cum_t - cs[e]) : 0.f;
              if (i < 8) m0[i] = v; else m1[i - 8] = v;
            }
          }
        }
        ssd_st8(smem + kSsdOffM + hf * 128 * 128 + ro[2 * m], m0);
        ssd_st8(smem + kSsdOffM + hf * 128 * 128 + ro[2 * m + 1], m1);
      }
      const __half2 e_t = __float2half2_rn(__expf(cum_t));
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        __half2 *hq = reinterpret_cast<__half2 *>(smem + kSsdOffCT + hf * 128 * 128 + ro[m]);
#pragma unroll
        for (int i = 0; i < 4; ++i) hq[i] = __hmul2(hq[i], e_t);
      }
      const float e_T = __expf(cum_T);
      float hv[16];
#pragma unroll
      for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
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

    // ---- y: row t = r, columns p of half hf, through a [p][t] bf16 tile (the products are
    // done with M), then 16-byte stores of whole row pieces
    {
      __nv_bfloat16 *ys = reinterpret_cast<__nv_bfloat16 *>(tmp);
      float yv[16];
#pragma unroll
      for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
        tc::tmem_ld16(t_Y + lane_base + cb * 16, yv);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) ys[(cb * 16 + i) * T + r] = __float2bfloat16_rn(yv[i]);
      }
      if (c == nchunks - 1 && args.h_last) {
        float hv[16];
#pragma unroll
        for (int cb = 2 * hf; cb < 2 * hf + 2; ++cb) {
          tc::tmem_ld16(t_H + lane_base + cb * 16, hv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) args.h_last[(bh * P + cb * 16 + i) * N + r] = hv[i];
        }
      }
      __syncthreads();
      const int p = tid >> 2, q = tid & 3;
      __nv_bfloat16 *yrow = args.y + (bh * P + p) * L + t0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int s0 = q * 32 + j * 8;
        const uint4 v = *reinterpret_cast<const uint4 *>(ys + p * T + s0);
        if (t0 + s0 + 8 <= L) {
          *reinterpret_cast<uint4 *>(yrow + s0) = v;
        } else {
          const __nv_bfloat16 *e = reinterpret_cast<const __nv_bfloat16 *>(&v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            if (t0 + s0 + i < L) yrow[s0 + i] = e[i];
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
