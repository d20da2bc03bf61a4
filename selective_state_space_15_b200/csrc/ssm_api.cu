// C ABI of the selective-scan library: argument checks, kernel selection, launches.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "ssm_scan.h"
#include "chunk_scan.cuh"
#include "state_update.cuh"

namespace {

using ssm::ScanArgs;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Tile shapes per state size: KI steps per lane, SPW segment lanes per channel, CPW channels
// per warp, WARPS warps per CTA.  Larger states get shorter chunks to bound shared memory.
template <int N> struct Shape;
template <> struct Shape<16> { static constexpr int KI = 16, SPW = 16, CPW = 2, WARPS = 8; };
template <> struct Shape<32> { static constexpr int KI = 16, SPW = 8, CPW = 4, WARPS = 8; };
template <> struct Shape<64> { static constexpr int KI = 8, SPW = 8, CPW = 4, WARPS = 8; };
template <> struct Shape<128> { static constexpr int KI = 8, SPW = 4, CPW = 8, WARPS = 4; };

template <typename T, typename TO, int N, bool HAS_Z, bool VEC>
ssm_status_t launch_chunk(const ScanArgs &a, cudaStream_t stream) {
  using S = Shape<N>;
  using Cfg = ssm::ChunkCfg<T, N, S::KI, S::SPW, S::CPW, S::WARPS>;
  auto kern = ssm::chunk_scan_kernel<T, TO, N, S::KI, S::SPW, S::CPW, S::WARPS, HAS_Z, VEC>;
  static bool configured = false;  // per instantiation; the attribute is per device function
  if (!configured) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kSmemBytes)) !=
        cudaSuccess)
      return SSM_ERR_CUDA;
    configured = true;
  }
  const int64_t blocks = int64_t(a.nseq) * a.ntiles;
  if (blocks == 0) return SSM_OK;
  if (blocks > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  kern<<<unsigned(blocks), Cfg::kThreads, Cfg::kSmemBytes, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <typename T, typename TO, int N>
ssm_status_t dispatch_zv(const ScanArgs &a, bool has_z, bool vec, cudaStream_t st) {
  if (has_z) return vec ? launch_chunk<T, TO, N, true, true>(a, st) : launch_chunk<T, TO, N, true, false>(a, st);
  return vec ? launch_chunk<T, TO, N, false, true>(a, st) : launch_chunk<T, TO, N, false, false>(a, st);
}

template <typename T, typename TO>
ssm_status_t dispatch_n(const ScanArgs &a, int N, bool has_z, bool vec, cudaStream_t st) {
  switch (N) {
    case 16: return dispatch_zv<T, TO, 16>(a, has_z, vec, st);
    case 32: return dispatch_zv<T, TO, 32>(a, has_z, vec, st);
    case 64: return dispatch_zv<T, TO, 64>(a, has_z, vec, st);
    case 128: return dispatch_zv<T, TO, 128>(a, has_z, vec, st);
    default: return SSM_ERR_UNSUPPORTED;
  }
}

int tile_channels(int N) {
  switch (N) {
    case 16: return Shape<16>::CPW * Shape<16>::WARPS;
    case 32: return Shape<32>::CPW * Shape<32>::WARPS;
    case 64: return Shape<64>::CPW * Shape<64>::WARPS;
    case 128: return Shape<128>::CPW * Shape<128>::WARPS;
    default: return 0;
  }
}

size_t elem_size(ssm_dtype_t t) { return t == SSM_BF16 ? 2 : 4; }

// Common checks for both scan entry points; fills `a` (except cu_seqlens / nseq).
ssm_status_t prepare_scan(const ssm_scan_params *p, bool varlen, ScanArgs &a, bool &vec) {
  if (!p) return SSM_ERR_INVALID_ARG;
  if (p->dtype != SSM_F32 && p->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (p->dim <= 0 || p->dstate <= 0 || p->seqlen < 0 || p->batch < 0) return SSM_ERR_INVALID_ARG;
  if (varlen && p->batch != 1) return SSM_ERR_INVALID_ARG;
  if (!p->u || !p->delta || !p->B || !p->C || !p->A || !p->y) return SSM_ERR_INVALID_ARG;
  if (tile_channels(int(p->dstate)) == 0 || p->dstate != int64_t(int(p->dstate))) return SSM_ERR_UNSUPPORTED;
  if (p->dim > (int64_t(1) << 31) || p->seqlen > (int64_t(1) << 40)) return SSM_ERR_UNSUPPORTED;
  a = ScanArgs{};
  a.u = p->u; a.delta = p->delta; a.z = p->z; a.B = p->B; a.C = p->C;
  a.A = p->A; a.Dskip = p->Dskip; a.bias = p->delta_bias; a.h0 = p->h0;
  a.y = p->y; a.h_last = p->h_last;
  a.dim = p->dim; a.seqlen = p->seqlen;
  a.x_dim_stride = p->x_dim_stride ? p->x_dim_stride : p->seqlen;
  a.x_batch_stride = p->x_batch_stride ? p->x_batch_stride : p->dim * a.x_dim_stride;
  a.bc_state_stride = p->bc_state_stride ? p->bc_state_stride : p->seqlen;
  a.bc_batch_stride = p->bc_batch_stride ? p->bc_batch_stride : p->dstate * a.bc_state_stride;
  if (a.x_dim_stride < p->seqlen || a.bc_state_stride < p->seqlen) return SSM_ERR_INVALID_ARG;
  if (!varlen && p->batch > 1 && (a.x_batch_stride < p->dim * a.x_dim_stride ||
                                  a.bc_batch_stride < p->dstate * a.bc_state_stride))
    return SSM_ERR_INVALID_ARG;
  const size_t es = elem_size(p->dtype);
  const int64_t V = int64_t(16 / es);
  vec = aligned16(p->u) && aligned16(p->delta) && aligned16(p->B) && aligned16(p->C) && aligned16(p->y) &&
        (!p->z || aligned16(p->z)) && a.x_dim_stride % V == 0 && a.bc_state_stride % V == 0 &&
        (varlen || (a.x_batch_stride % V == 0 && a.bc_batch_stride % V == 0));
  a.ntiles = int((p->dim + tile_channels(int(p->dstate)) - 1) / tile_channels(int(p->dstate)));
  return SSM_OK;
}

ssm_status_t run_scan(const ScanArgs &a, ssm_dtype_t dt, bool y_fp32, int N, bool vec, cudaStream_t st) {
  const bool has_z = a.z != nullptr;
  if (dt == SSM_BF16) {
    if (y_fp32) return dispatch_n<__nv_bfloat16, float>(a, N, has_z, vec, st);
    return dispatch_n<__nv_bfloat16, __nv_bfloat16>(a, N, has_z, vec, st);
  }
  return dispatch_n<float, float>(a, N, has_z, vec, st);
}

}  // namespace

extern "C" {

ssm_status_t ssm_scan_fwd(const ssm_scan_params *p, void *workspace, size_t workspace_bytes,
                          ssm_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, false, a, vec);
  if (st != SSM_OK) return st;
  if (p->batch == 0) return SSM_OK;
  if (p->batch > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  a.cu_seqlens = nullptr;
  a.nseq = int(p->batch);
  return run_scan(a, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_scan_fwd_varlen(const ssm_scan_params *p, const int32_t *cu_seqlens, int64_t nseq,
                                 void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!cu_seqlens || nseq < 0) return SSM_ERR_INVALID_ARG;
  if (nseq > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  if (p && p->seqlen > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;  // int32 offsets
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, true, a, vec);
  if (st != SSM_OK) return st;
  if (nseq == 0) return SSM_OK;
  a.cu_seqlens = cu_seqlens;
  a.nseq = int(nseq);
  return run_scan(a, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_state_update(float *pool, int64_t num_slots, const int32_t *slot_ids, int64_t R,
                              const ssm_scan_params *p, ssm_stream_t stream) {
  if (!p || !pool || !slot_ids || num_slots <= 0 || R < 0) return SSM_ERR_INVALID_ARG;
  if (p->dtype != SSM_F32 && p->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (p->batch != R || p->seqlen != 1 || p->dim <= 0 || p->dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (!p->u || !p->delta || !p->B || !p->C || !p->A || !p->y) return SSM_ERR_INVALID_ARG;
  const int64_t N = p->dstate;
  if (N % 4 != 0 || N > 128) return SSM_ERR_UNSUPPORTED;
  int qlog2 = 0;
  while ((int64_t(4) << qlog2) < N) ++qlog2;
  if ((int64_t(4) << qlog2) != N) return SSM_ERR_UNSUPPORTED;  // dstate/4 must be a power of two
  if (!aligned16(pool) || !aligned16(p->A)) return SSM_ERR_INVALID_ARG;
  if (R == 0) return SSM_OK;
  ssm::UpdateArgs a{};
  a.pool = pool; a.slot_ids = slot_ids;
  a.u = p->u; a.delta = p->delta; a.z = p->z; a.B = p->B; a.C = p->C;
  a.A = p->A; a.Dskip = p->Dskip; a.bias = p->delta_bias; a.y = p->y;
  a.num_slots = num_slots; a.R = R; a.dim = p->dim;
  a.x_stride = p->x_batch_stride ? p->x_batch_stride : p->dim;
  a.bc_stride = p->bc_batch_stride ? p->bc_batch_stride : N;
  if (a.x_stride < p->dim || a.bc_stride < N) return SSM_ERR_INVALID_ARG;
  a.dstate = int(N);
  a.qlog2 = qlog2;
  const int64_t threads = R * p->dim * (N / 4);
  const int64_t blocks = (threads + 255) / 256;
  if (blocks > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool has_z = p->z != nullptr;
  using bf16 = __nv_bfloat16;
  if (p->dtype == SSM_BF16 && !p->y_fp32) {
    if (has_z) ssm::state_update_kernel<bf16, bf16, true><<<unsigned(blocks), 256, 0, st>>>(a);
    else ssm::state_update_kernel<bf16, bf16, false><<<unsigned(blocks), 256, 0, st>>>(a);
  } else if (p->dtype == SSM_BF16) {
    if (has_z) ssm::state_update_kernel<bf16, float, true><<<unsigned(blocks), 256, 0, st>>>(a);
    else ssm::state_update_kernel<bf16, float, false><<<unsigned(blocks), 256, 0, st>>>(a);
  } else {
    if (has_z) ssm::state_update_kernel<float, float, true><<<unsigned(blocks), 256, 0, st>>>(a);
    else ssm::state_update_kernel<float, float, false><<<unsigned(blocks), 256, 0, st>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

size_t ssm_scan_workspace_size(const ssm_scan_params *p, int64_t nseq) {
  (void)p;
  (void)nseq;
  return 0;
}

ssm_status_t ssm_get_device_status(ssm_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, ssm::g_status, sizeof(int)) != cudaSuccess) return SSM_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(ssm::g_status, &zero, sizeof(int)) != cudaSuccess) return SSM_ERR_CUDA;
  return static_cast<ssm_status_t>(v);
}

const char *ssm_status_string(ssm_status_t s) {
  switch (s) {
    case SSM_OK: return "SSM_OK";
    case SSM_ERR_INVALID_ARG: return "SSM_ERR_INVALID_ARG";
    case SSM_ERR_UNSUPPORTED: return "SSM_ERR_UNSUPPORTED";
    case SSM_ERR_CUDA: return "SSM_ERR_CUDA";
    case SSM_ERR_BAD_SLOT: return "SSM_ERR_BAD_SLOT";
    case SSM_ERR_TIMEOUT: return "SSM_ERR_TIMEOUT";
    case SSM_ERR_WORKSPACE: return "SSM_ERR_WORKSPACE";
    default: return "SSM_ERR_UNKNOWN";
  }
}

int ssm_abi_version(void) { return SSM_ABI_VERSION; }

}  // extern "C"
