// C ABI of the selective-scan library: argument checks, kernel selection, launches.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <utility>

#include "ssm_scan.h"
#include "chunk_scan.cuh"
#include "seq_scan.cuh"
#include "seq_bwd.cuh"
#include "ssd_chunk.cuh"
#include "state_update.cuh"

namespace {

using ssm::ScanArgs;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// Per (kernel, device) launch facts: the dynamic shared-memory attribute is set and the
// occupancy queried once per device, under a lock, so host threads that drive different
// GPUs (or the same one) can launch concurrently.
struct LaunchInfo {
  ssm_status_t status = SSM_OK;
  int blocks_per_sm = 0;
  int num_sms = 0;
};
std::mutex g_launch_mutex;
std::map<std::pair<const void *, int>, LaunchInfo> g_launch_info;

ssm_status_t launch_info(const void *kern, int threads, size_t smem, LaunchInfo &out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SSM_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_launch_mutex);
  auto it = g_launch_info.find({kern, dev});
  if (it == g_launch_info.end()) {
    LaunchInfo li;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&li.blocks_per_sm, kern, threads, smem) != cudaSuccess ||
        cudaDeviceGetAttribute(&li.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      li.status = SSM_ERR_CUDA;
    }
    if (li.blocks_per_sm < 1) li.blocks_per_sm = 1;
    it = g_launch_info.emplace(std::make_pair(kern, dev), li).first;
  }
  out = it->second;
  return out.status;
}

// Tile shapes: KI steps per lane, SPW segment lanes per channel, CPW channels per warp, CW
// channel warps and NG state groups per CTA; when CPW * SPW < 32 the lanes of a warp form
// 32 / (CPW * SPW) groups that split the states as well.  Larger states get shorter chunks
// to bound shared memory; the narrow shapes split the states for parallelism (N=16: two
// lane groups of one channel per warp; N=128: 16 warps).  32-bit inputs can take a shape of
// their own (F32): the narrow N=16 one halves the chunk so that four CTAs fit per SM.
struct ShapeInfo {
  int KI, SPW, CPW, CW, NG;
  int ct() const { return CPW * CW; }
  int tc() const { return SPW * KI; }
};
template <int N, bool NARROW, bool F32 = false> struct Shape;
template <int N, bool NARROW> struct Shape<N, NARROW, true> : Shape<N, NARROW, false> {};
template <> struct Shape<16, false> { static constexpr int KI = 16, SPW = 4, CPW = 8, CW = 4, NG = 1; };
// Narrow N=16 tile for 16-bit inputs: 16 segments x 2 lane groups (8 states each) of one channel
// per warp, 256-step chunks, B/C converted in the state loop.  SSM_NARROW16_LG = 4 builds 8
// segments x 4 lane groups (4 states each), 128-step chunks with B/C widened to float32 once per
// chunk: measured 35 % slower on a 131072-step sequence of 2560 channels (4.43 vs 3.29 ms).
#ifndef SSM_NARROW16_LG
#define SSM_NARROW16_LG 2
#endif
template <> struct Shape<16, true> {
  static constexpr int KI = 16, SPW = SSM_NARROW16_LG == 4 ? 8 : 16, CPW = 1, CW = 4, NG = 1;
};
template <> struct Shape<16, true, true> { static constexpr int KI = 8, SPW = 16, CPW = 1, CW = 4, NG = 1; };
template <> struct Shape<32, false> { static constexpr int KI = 16, SPW = 8, CPW = 4, CW = 8, NG = 1; };
template <> struct Shape<64, false> { static constexpr int KI = 8, SPW = 8, CPW = 4, CW = 8, NG = 1; };
template <> struct Shape<128, false> { static constexpr int KI = 8, SPW = 4, CPW = 8, CW = 4, NG = 1; };
template <> struct Shape<128, true> { static constexpr int KI = 16, SPW = 8, CPW = 4, CW = 1, NG = 16; };
// N=256: 8 warps share an 8-channel tile and take 32 states each (per-(channel, state) arrays
// and the B/C chunk of a wider tile would not fit in shared memory)
template <> struct Shape<256, false> { static constexpr int KI = 8, SPW = 4, CPW = 8, CW = 1, NG = 8; };
template <int N, bool NARROW, bool F32> ShapeInfo shape_of() {
  using S = Shape<N, NARROW, F32>;
  return ShapeInfo{S::KI, S::SPW, S::CPW, S::CW, S::NG};
}
bool shape_for(int N, bool narrow, bool f32, ShapeInfo &si) {
  switch (N) {
    case 16:
      si = narrow ? (f32 ? shape_of<16, true, true>() : shape_of<16, true, false>()) : shape_of<16, false, false>();
      return true;
    case 32: si = shape_of<32, false, false>(); return true;
    case 64: si = shape_of<64, false, false>(); return true;
    case 128: si = narrow ? shape_of<128, true, false>() : shape_of<128, false, false>(); return true;
    case 256: si = shape_of<256, false, false>(); return true;
    default: return false;
  }
}

// How a scan is run: persistent ticketed units for 16-byte aligned fixed-length batches,
// one CTA per (sequence, tile) otherwise.
struct Plan {
  bool persist = false, narrow = false;
  bool seq = false;  // lane-sequential kernel (seq_scan.cuh) instead of the chunked one
  ShapeInfo si{};
  int64_t ntiles = 0, nchains = 0, nchunks = 0;
  size_t flags_off = 0, carries_off = 0, ws_bytes = 0;
};
// batch * dim below these: split the states over several warps (N=16: 2, N=128: 16; the
// N=128 narrow tile is planned for 16-bit inputs only, whose B/C chunk fits in shared memory)
constexpr int64_t kNarrowChannels16 = 8192, kNarrowChannels128 = 32768;

int64_t groups_of(const ssm_scan_params *p) { return p->ngroups > 1 ? p->ngroups : 1; }

// Test hook (ssm_test_drop_first_handoff): consumed by the next persistent launch.
std::atomic<bool> g_test_drop_first_handoff{false};

// Lane-sequential kernel: lanes per channel (LPC: 4 lanes of 4 states for dstate 16, of 8
// for dstate 32; a CTA of four warps then holds 32 channels), the resident CTAs per SM it is
// launched with (0: as many as fit), and the number of (sequence, channel) pairs from which
// AUTO prefers it.  Units are (sequence, 32-channel tile) pairs, about twice as many as CTA
// slots on the packed workloads, so that the longest-first ticket can even out the tail.
#ifndef SSM_SEQ_LPC16
#define SSM_SEQ_LPC16 4
#endif
#ifndef SSM_SEQ_MAX_CTAS
#define SSM_SEQ_MAX_CTAS 0
#endif
#ifndef SSM_SEQ_WARPS
#define SSM_SEQ_WARPS 4
#endif
constexpr int seq_lpc(int N) { return N == 16 ? SSM_SEQ_LPC16 : 4; }
constexpr int kSeqWarps = SSM_SEQ_WARPS;
constexpr int kSeqMaxCtasPerSm = SSM_SEQ_MAX_CTAS;
// AUTO: measured on B200, the chunked kernel is the faster of the two on every workload here
// (packed bf16 batch of 16 x 2048: 0.50 vs 0.53 ms), so AUTO takes it; the sequential kernel
// is chosen explicitly.
constexpr int64_t kSeqMinPairs = int64_t(1) << 62;
bool seq_supported(const ssm_scan_params *p, bool vec) {
  return vec && (p->dstate == 16 || p->dstate == 32) && p->discretization == SSM_DISC_EULER;
}

// Returns false when the requested algorithm has no kernel for this problem.
bool make_plan(const ssm_scan_params *p, int64_t nseq, bool varlen, bool vec, Plan &pl) {
  const int N = int(p->dstate);
  const int64_t dim = p->dim, seqlen = p->seqlen;
  const bool bf16 = p->dtype == SSM_BF16;
  pl = Plan{};
  if (p->algorithm == SSM_ALGO_SEQUENTIAL ||
      (p->algorithm == SSM_ALGO_AUTO && seq_supported(p, vec) && nseq * dim >= kSeqMinPairs)) {
    if (!seq_supported(p, vec)) return false;
    pl.seq = true;
    const int64_t G = groups_of(p);
    const int64_t ct = int64_t(kSeqWarps) * (32 / seq_lpc(N));
    pl.ntiles = G * ((dim / G + ct - 1) / ct);
    pl.nchains = nseq * pl.ntiles;
    pl.ws_bytes = 16;  // the unit ticket
    return true;
  }
  pl.persist = !varlen && vec && seqlen > 0;
  pl.narrow = pl.persist && ((N == 16 && nseq * dim < kNarrowChannels16) ||
                             (N == 128 && bf16 && nseq * dim < kNarrowChannels128));
  if (!shape_for(N, pl.narrow, p->dtype == SSM_F32, pl.si)) return false;
  // channel tiles never straddle a group of channels
  const int64_t G = groups_of(p);
  pl.ntiles = G * ((dim / G + pl.si.ct() - 1) / pl.si.ct());
  pl.nchains = nseq * pl.ntiles;
  pl.nchunks = pl.persist ? (seqlen + pl.si.tc() - 1) / pl.si.tc() : 0;
  if (pl.persist) {
    pl.flags_off = 16;  // the ticket counter lives in the first 16 bytes
    pl.carries_off = (pl.flags_off + size_t(pl.nchains) * 4 + 15) / 16 * 16;
    pl.ws_bytes = pl.carries_off + size_t(pl.nchains) * pl.si.ct() * N * sizeof(float);
  }
  return true;
}

template <typename T, typename TO, int N, bool NARROW, bool HAS_Z, bool VEC, bool PERSIST, bool ZOH>
ssm_status_t launch_chunk(ScanArgs a, const Plan &pl, void *ws, cudaStream_t stream) {
  using S = Shape<N, NARROW, sizeof(T) == 4>;
  using Cfg = ssm::ChunkCfg<T, N, S::KI, S::SPW, S::CPW, S::CW, S::NG>;
  auto kern = ssm::chunk_scan_kernel<T, TO, N, S::KI, S::SPW, S::CPW, S::CW, S::NG, HAS_Z, VEC, PERSIST, ZOH>;
  constexpr size_t kSmem = Cfg::kSmemBytes + (ZOH ? Cfg::kInvABytes : 0);
  LaunchInfo li;
  if (launch_info(reinterpret_cast<const void *>(kern), Cfg::kThreads, kSmem, li) != SSM_OK) return SSM_ERR_CUDA;
  const int max_blocks_per_sm = li.blocks_per_sm, num_sms = li.num_sms;
  if (pl.nchains == 0) return SSM_OK;
  int64_t blocks = pl.nchains;
  if constexpr (PERSIST) {
    unsigned char *w = static_cast<unsigned char *>(ws);
    if (cudaMemsetAsync(w, 0, pl.carries_off, stream) != cudaSuccess) return SSM_ERR_CUDA;
    const int64_t resident = int64_t(num_sms) * (max_blocks_per_sm > 0 ? max_blocks_per_sm : 1);
    // The units of one chain run one after another, so splitting a chain only evens out the
    // load when there are more chains than CTA slots.  Then: enough units per slot for an even
    // spread (about 16), and at least kMinGroup chunks per unit to keep the per-unit overhead
    // (ticket, hand-off, first load) small; otherwise a chain is a single unit.
    constexpr int64_t kMinGroup = 6;
    int64_t group = pl.nchunks;
    if (pl.nchains > resident) {
      group = (pl.nchunks * pl.nchains) / (16 * resident);
      group = group < kMinGroup ? kMinGroup : group;
      group = group > pl.nchunks ? pl.nchunks : group;
    }
    const bool drop_first = g_test_drop_first_handoff.exchange(false);
    if (drop_first) group = 1;
    const int64_t ngroups = (pl.nchunks + group - 1) / group;
    if (pl.nchains * ngroups > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
    a.ticket = reinterpret_cast<uint32_t *>(w);
    a.flags = reinterpret_cast<uint32_t *>(w + pl.flags_off);
    a.carries = reinterpret_cast<float *>(w + pl.carries_off);
    a.nchains = int(pl.nchains);
    a.group = int(group);
    a.total_units = int(pl.nchains * ngroups);
    blocks = a.total_units < resident ? a.total_units : resident;
    if (drop_first) {  // the unit counter starts past the first chunk group
      const uint32_t start = uint32_t(pl.nchains);
      if (cudaMemcpyAsync(w, &start, sizeof(start), cudaMemcpyHostToDevice, stream) != cudaSuccess)
        return SSM_ERR_CUDA;
    }
  }
  if (blocks > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  kern<<<unsigned(blocks), Cfg::kThreads, kSmem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

// Lane-sequential kernel: a persistent grid over (sequence, channel tile) units taken from a
// ticket in the workspace (zeroed here, on the stream).
template <typename T, typename TO, int N, bool HAS_Z>
ssm_status_t launch_seq(ScanArgs a, const Plan &pl, void *ws, cudaStream_t stream) {
  constexpr int LPC = seq_lpc(N);
  constexpr int TC = sizeof(T) == 2 ? 32 : 16;  // 64-byte rows either way
  using Cfg = ssm::SeqCfg<T, N, LPC, TC, kSeqWarps>;
  auto kern = ssm::seq_scan_kernel<T, TO, N, LPC, TC, kSeqWarps, HAS_Z>;
  LaunchInfo li;
  if (launch_info(reinterpret_cast<const void *>(kern), Cfg::kThreads, Cfg::kSmemBytes, li) != SSM_OK)
    return SSM_ERR_CUDA;
  if (pl.nchains == 0) return SSM_OK;
  if (pl.nchains > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  if (cudaMemsetAsync(ws, 0, 16, stream) != cudaSuccess) return SSM_ERR_CUDA;
  a.ticket = static_cast<uint32_t *>(ws);
  a.total_units = int(pl.nchains);
  const int per_sm = kSeqMaxCtasPerSm > 0 && kSeqMaxCtasPerSm < li.blocks_per_sm ? kSeqMaxCtasPerSm : li.blocks_per_sm;
  const int64_t resident = int64_t(li.num_sms) * per_sm;
  const int64_t blocks = pl.nchains < resident ? pl.nchains : resident;
  kern<<<unsigned(blocks), Cfg::kThreads, Cfg::kSmemBytes, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

template <typename T, typename TO>
ssm_status_t dispatch_seq(const ScanArgs &a, const Plan &pl, int N, bool has_z, void *ws, cudaStream_t st) {
  switch (N) {
    case 16: return has_z ? launch_seq<T, TO, 16, true>(a, pl, ws, st) : launch_seq<T, TO, 16, false>(a, pl, ws, st);
    case 32: return has_z ? launch_seq<T, TO, 32, true>(a, pl, ws, st) : launch_seq<T, TO, 32, false>(a, pl, ws, st);
    default: return SSM_ERR_UNSUPPORTED;
  }
}

template <typename T, typename TO, int N, bool NARROW, bool ZOH>
ssm_status_t dispatch_zvp(const ScanArgs &a, const Plan &pl, bool has_z, bool vec, void *ws, cudaStream_t st) {
  if (pl.persist) {
    if (has_z) return launch_chunk<T, TO, N, NARROW, true, true, true, ZOH>(a, pl, ws, st);
    return launch_chunk<T, TO, N, NARROW, false, true, true, ZOH>(a, pl, ws, st);
  }
  if constexpr (NARROW) {
    return SSM_ERR_UNSUPPORTED;  // the narrow shape is only planned for persistent launches
  } else {
    if (has_z)
      return vec ? launch_chunk<T, TO, N, false, true, true, false, ZOH>(a, pl, ws, st)
                 : launch_chunk<T, TO, N, false, true, false, false, ZOH>(a, pl, ws, st);
    return vec ? launch_chunk<T, TO, N, false, false, true, false, ZOH>(a, pl, ws, st)
               : launch_chunk<T, TO, N, false, false, false, false, ZOH>(a, pl, ws, st);
  }
}

template <typename T, typename TO, bool ZOH>
ssm_status_t dispatch_n(const ScanArgs &a, const Plan &pl, int N, bool has_z, bool vec, void *ws,
                        cudaStream_t st) {
  switch (N) {
    case 16: return pl.narrow ? dispatch_zvp<T, TO, 16, true, ZOH>(a, pl, has_z, vec, ws, st)
                              : dispatch_zvp<T, TO, 16, false, ZOH>(a, pl, has_z, vec, ws, st);
    case 32: return dispatch_zvp<T, TO, 32, false, ZOH>(a, pl, has_z, vec, ws, st);
    case 64: return dispatch_zvp<T, TO, 64, false, ZOH>(a, pl, has_z, vec, ws, st);
    case 128:
      if constexpr (std::is_same<T, float>::value) {
        return dispatch_zvp<T, TO, 128, false, ZOH>(a, pl, has_z, vec, ws, st);  // no narrow plan for float32
      } else {
        return pl.narrow ? dispatch_zvp<T, TO, 128, true, ZOH>(a, pl, has_z, vec, ws, st)
                         : dispatch_zvp<T, TO, 128, false, ZOH>(a, pl, has_z, vec, ws, st);
      }
    case 256: return dispatch_zvp<T, TO, 256, false, ZOH>(a, pl, has_z, vec, ws, st);
    default: return SSM_ERR_UNSUPPORTED;
  }
}

template <typename T, typename TO>
ssm_status_t dispatch_disc(const ScanArgs &a, const Plan &pl, int N, bool has_z, bool vec, bool zoh, void *ws,
                           cudaStream_t st) {
  return zoh ? dispatch_n<T, TO, true>(a, pl, N, has_z, vec, ws, st)
             : dispatch_n<T, TO, false>(a, pl, N, has_z, vec, ws, st);
}

size_t elem_size(ssm_dtype_t t) { return t == SSM_BF16 ? 2 : 4; }

// Common checks for the scan entry points; fills `a` (except cu_seqlens / nseq).  The backward
// reads the forward's description but writes no y (need_y = false).
ssm_status_t prepare_scan(const ssm_scan_params *p, bool varlen, ScanArgs &a, bool &vec, bool need_y = true) {
  if (!p) return SSM_ERR_INVALID_ARG;
  if (p->dtype != SSM_F32 && p->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (p->discretization != SSM_DISC_EULER && p->discretization != SSM_DISC_ZOH) return SSM_ERR_INVALID_ARG;
  if (p->algorithm != SSM_ALGO_AUTO && p->algorithm != SSM_ALGO_CHUNKED && p->algorithm != SSM_ALGO_SEQUENTIAL)
    return SSM_ERR_INVALID_ARG;
  if (p->dim <= 0 || p->dstate <= 0 || p->seqlen < 0 || p->batch < 0) return SSM_ERR_INVALID_ARG;
  if (varlen && p->batch != 1) return SSM_ERR_INVALID_ARG;
  if (!p->u || !p->delta || !p->B || !p->C || !p->A || (need_y && !p->y)) return SSM_ERR_INVALID_ARG;
  ShapeInfo probe;
  if (p->dstate > 256 || !shape_for(int(p->dstate), false, false, probe)) return SSM_ERR_UNSUPPORTED;
  if (p->dim > (int64_t(1) << 31) || p->seqlen > (int64_t(1) << 40)) return SSM_ERR_UNSUPPORTED;
  a = ScanArgs{};
  a.u = p->u; a.delta = p->delta; a.z = p->z; a.B = p->B; a.C = p->C;
  a.A = p->A; a.Dskip = p->Dskip; a.bias = p->delta_bias; a.h0 = p->h0;
  a.y = p->y; a.h_last = p->h_last;
  a.dim = p->dim; a.seqlen = p->seqlen;
  a.x_dim_stride = p->x_dim_stride ? p->x_dim_stride : p->seqlen;
  a.x_batch_stride = p->x_batch_stride ? p->x_batch_stride : p->dim * a.x_dim_stride;
  a.bc_state_stride = p->bc_state_stride ? p->bc_state_stride : p->seqlen;
  if (p->ngroups < 0 || p->bc_group_stride < 0) return SSM_ERR_INVALID_ARG;
  const int64_t G = groups_of(p);
  if (p->dim % G != 0) return SSM_ERR_INVALID_ARG;
  a.group_dim = p->dim / G;
  a.bc_group_stride = p->bc_group_stride ? p->bc_group_stride : p->dstate * a.bc_state_stride;
  if (G > 1 && a.bc_group_stride < p->dstate * a.bc_state_stride) return SSM_ERR_INVALID_ARG;
  a.bc_batch_stride = p->bc_batch_stride ? p->bc_batch_stride : G * a.bc_group_stride;
  if (a.x_dim_stride < p->seqlen || a.bc_state_stride < p->seqlen) return SSM_ERR_INVALID_ARG;
  if (!varlen && p->batch > 1 && (a.x_batch_stride < p->dim * a.x_dim_stride ||
                                  a.bc_batch_stride < G * p->dstate * a.bc_state_stride))
    return SSM_ERR_INVALID_ARG;
  const size_t es = elem_size(p->dtype);
  const int64_t V = int64_t(16 / es);
  vec = aligned16(p->u) && aligned16(p->delta) && aligned16(p->B) && aligned16(p->C) && aligned16(p->y) &&
        (!p->z || aligned16(p->z)) && a.x_dim_stride % V == 0 && a.bc_state_stride % V == 0 &&
        a.bc_group_stride % V == 0 &&
        (varlen || (a.x_batch_stride % V == 0 && a.bc_batch_stride % V == 0));
  return SSM_OK;
}

ssm_status_t run_scan(ScanArgs a, const Plan &pl, ssm_dtype_t dt, bool y_fp32, int N, bool vec, bool zoh,
                      void *ws, size_t ws_bytes, cudaStream_t st) {
  if (pl.ws_bytes > 0 && (ws == nullptr || ws_bytes < pl.ws_bytes || (reinterpret_cast<uintptr_t>(ws) & 15)))
    return SSM_ERR_WORKSPACE;
  if (pl.ntiles > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  a.ntiles = int(pl.ntiles);
  a.tiles_per_group = int(pl.ntiles / (a.dim / a.group_dim));
  const bool has_z = a.z != nullptr;
  if (pl.seq) {
    if (dt == SSM_BF16)
      return y_fp32 ? dispatch_seq<__nv_bfloat16, float>(a, pl, N, has_z, ws, st)
                    : dispatch_seq<__nv_bfloat16, __nv_bfloat16>(a, pl, N, has_z, ws, st);
    return dispatch_seq<float, float>(a, pl, N, has_z, ws, st);
  }
  if (dt == SSM_BF16) {
    if (y_fp32) return dispatch_disc<__nv_bfloat16, float>(a, pl, N, has_z, vec, zoh, ws, st);
    return dispatch_disc<__nv_bfloat16, __nv_bfloat16>(a, pl, N, has_z, vec, zoh, ws, st);
  }
  return dispatch_disc<float, float>(a, pl, N, has_z, vec, zoh, ws, st);
}

// Scratch for ssm_scan_fwd_noalloc: a static device array that every GPU loading the
// library holds until the process exits.  In host code `g_noalloc_scratch` names a host-side
// stand-in, not device memory, so its device address is looked up once per device.
constexpr size_t kNoAllocScratchBytes = SSM_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void *g_noalloc_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device (looked up on first use).
ssm_status_t noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return SSM_ERR_CUDA;
  if (dev >= kMaxDevices) return SSM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return SSM_ERR_CUDA;
    g_noalloc_addr[dev] = ptr;
  }
  *out = g_noalloc_addr[dev];
  return SSM_OK;
}

// Decode launches: the N = 16 kernel (pool slices streamed by bulk copies), else G states per
// thread.
template <typename T, typename TO, bool ZOH>
ssm_status_t launch_update_disc(const ssm::UpdateArgs &a, int G, bool has_z, dim3 blocks, cudaStream_t st) {
  using namespace ssm;
  if (a.dstate == 16) {
    // one block per (channel group, residue class of requests): as many request classes as
    // keep every resident block slot busy
    auto kern = has_z ? state_update16_bulk_kernel<T, TO, true, ZOH> : state_update16_bulk_kernel<T, TO, false, ZOH>;
    LaunchInfo li;
    if (launch_info(reinterpret_cast<const void *>(kern), kUpdateThreads, kUpdBulkSmem, li) != SSM_OK)
      return SSM_ERR_CUDA;
    const int64_t ngrp = (a.dim + kUpdBulkCh - 1) / kUpdBulkCh;
    const int64_t slots = int64_t(li.num_sms) * li.blocks_per_sm;
    const int64_t nrb = std::min<int64_t>(std::max<int64_t>(1, std::min<int64_t>(a.R, slots / ngrp)), 65535);
    kern<<<dim3(unsigned(ngrp), unsigned(nrb)), kUpdateThreads, kUpdBulkSmem, st>>>(a);
    return SSM_OK;
  }
  auto go = [&](auto g_tag) {
    constexpr int GG = decltype(g_tag)::value;
    if (has_z) state_update_kernel<T, TO, true, GG, ZOH><<<blocks, kUpdateThreads, 0, st>>>(a);
    else state_update_kernel<T, TO, false, GG, ZOH><<<blocks, kUpdateThreads, 0, st>>>(a);
  };
  if (G == 16) go(std::integral_constant<int, 16>{});
  else if (G == 8) go(std::integral_constant<int, 8>{});
  else go(std::integral_constant<int, 4>{});
  return SSM_OK;
}
template <typename T, typename TO>
ssm_status_t launch_update(const ssm::UpdateArgs &a, int G, bool has_z, bool zoh, dim3 blocks, cudaStream_t st) {
  return zoh ? launch_update_disc<T, TO, true>(a, G, has_z, blocks, st)
             : launch_update_disc<T, TO, false>(a, G, has_z, blocks, st);
}

// ---- backward (ssm_scan_bwd) ----
// Units are (sequence, time segment, tile of 32 channels), segments whole chunks, at least
// kBwdMinSegChunks chunks long and otherwise as long as still gives kBwdUnitsWanted units.
// Workspace (float32 unless noted): two unit tickets (16 bytes each), the block checkpoints
// [batch][nblk][dim][N], the per-block Delta sums [batch][nblk][dim], the per-segment Delta
// sums [batch][nseg][dim] and the two per-segment state arrays [batch][nseg][dim][N].
constexpr int kBwdTC16 = 32;  // chunk of the backward kernels for 16-bit inputs (64-byte rows)
#ifndef SSM_BWD_TC_F32
#define SSM_BWD_TC_F32 32
#endif
constexpr int kBwdTC32 = SSM_BWD_TC_F32;  // the same for float32 inputs (128-byte rows; 72 KB, 3 CTAs per SM)
constexpr int kBwdWarps = 4;  // warps per CTA (8 channels each)
#ifndef SSM_BWD_UNITS_PER_SM
#define SSM_BWD_UNITS_PER_SM 32  // backward units wanted per SM: long sequences cut into more segments balance better
#endif
#ifndef SSM_BWD_MIN_SEG_CHUNKS
#define SSM_BWD_MIN_SEG_CHUNKS 4
#endif
constexpr int64_t kBwdUnitsWanted = SSM_BWD_UNITS_PER_SM * 148;
constexpr int64_t kBwdMinSegChunks = SSM_BWD_MIN_SEG_CHUNKS;
struct BwdPlan {
  int64_t nblk = 0, ntiles = 0, nseg = 0, seg_len = 0, nunits = 0;
  size_t off_ckpt = 0, off_cumd = 0, off_ssum = 0, off_sh = 0, off_sg = 0, bytes = 0;
};
bool make_bwd_plan(const ssm_scan_params *p, bool vec, BwdPlan &bp) {
  if (!vec || p->dstate != 16 || groups_of(p) != 1) return false;
  const int64_t TC = p->dtype == SSM_F32 ? kBwdTC32 : kBwdTC16;
  const int64_t CT = 8 * kBwdWarps, L = p->seqlen, N = p->dstate;
  bp.nblk = (L + 7) / 8;
  bp.ntiles = (p->dim + CT - 1) / CT;
  const int64_t chunks = std::max<int64_t>(1, (L + TC - 1) / TC);
  const int64_t rows = std::max<int64_t>(1, p->batch * bp.ntiles);
  const int64_t want_seg = (kBwdUnitsWanted + rows - 1) / rows;  // segments per sequence wanted
  const int64_t seg_chunks = std::max<int64_t>(kBwdMinSegChunks, chunks / std::max<int64_t>(1, want_seg));
  bp.seg_len = seg_chunks * TC;
  bp.nseg = std::max<int64_t>(1, (L + bp.seg_len - 1) / bp.seg_len);
  bp.nunits = p->batch * bp.nseg * bp.ntiles;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t f = sizeof(float), B = size_t(p->batch), D = size_t(p->dim);
  bp.off_ckpt = 256;
  bp.off_cumd = al(bp.off_ckpt + B * bp.nblk * D * N * f);
  bp.off_ssum = al(bp.off_cumd + B * bp.nblk * D * f);
  bp.off_sh = al(bp.off_ssum + B * bp.nseg * D * f);
  bp.off_sg = al(bp.off_sh + B * bp.nseg * D * N * f);
  bp.bytes = bp.off_sg + B * bp.nseg * D * N * f;
  return true;
}

template <typename X> struct TypeTag { using type = X; };

template <typename T, typename TG, bool HAS_Z, bool ZOH>
ssm_status_t launch_bwd(ScanArgs a, const ssm::BwdArgs &bwa, const BwdPlan &bp, const ssm_scan_params *p,
                        unsigned char *ws, cudaStream_t st) {
  constexpr int N = 16, W = kBwdWarps;
  constexpr int TC = sizeof(T) == 2 ? kBwdTC16 : kBwdTC32;
  using Cfg = ssm::BwdCfg<T, TG, N, TC, W>;
  a.ntiles = int(bp.ntiles);
  a.nseq = int(p->batch);
  a.total_units = int(bp.nunits);
  // 1. the segment pass
  {
    auto kern = ssm::bwd_seg_kernel<T, TG, N, TC, W, HAS_Z, ZOH>;
    LaunchInfo li;
    if (launch_info(reinterpret_cast<const void *>(kern), Cfg::kThreads, Cfg::kSegSmemBytes, li) != SSM_OK)
      return SSM_ERR_CUDA;
    ScanArgs f = a;
    f.ticket = reinterpret_cast<uint32_t *>(ws);
    const int64_t blocks = std::min<int64_t>(bp.nunits, int64_t(li.num_sms) * li.blocks_per_sm);
    kern<<<unsigned(blocks), Cfg::kThreads, Cfg::kSegSmemBytes, st>>>(f, bwa);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
  }
  // 2. the segment scan
  {
    const int64_t n = p->batch * p->dim * N;
    ssm::bwd_seg_scan_kernel<<<unsigned((n + 255) / 256), 256, 0, st>>>(
        p->A, p->h0, bwa.dh_last, bwa.seg_sum, bwa.seg_h, bwa.seg_g, p->batch, p->dim, N, int(bp.nseg));
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
  }
  // 3. the walk
  {
    auto kern = ssm::seq_bwd_kernel<T, TG, N, TC, W, HAS_Z, ZOH>;
    LaunchInfo li;
    if (launch_info(reinterpret_cast<const void *>(kern), Cfg::kThreads, Cfg::kSmemBytes, li) != SSM_OK)
      return SSM_ERR_CUDA;
    ScanArgs b = a;
    b.ticket = reinterpret_cast<uint32_t *>(ws + 16);
    const int64_t blocks = std::min<int64_t>(bp.nunits, int64_t(li.num_sms) * li.blocks_per_sm);
    kern<<<unsigned(blocks), Cfg::kThreads, Cfg::kSmemBytes, st>>>(b, bwa);
    if (cudaGetLastError() != cudaSuccess) return SSM_ERR_CUDA;
  }
  return SSM_OK;
}

}  // namespace

extern "C" {

ssm_status_t ssm_scan_fwd_noalloc(const ssm_scan_params *p, ssm_stream_t stream) {
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, false, a, vec);
  if (st != SSM_OK) return st;
  if (p->batch == 0) return SSM_OK;
  if (p->batch > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  Plan pl;
  if (!make_plan(p, p->batch, false, vec, pl)) return SSM_ERR_UNSUPPORTED;
  if (pl.ws_bytes > kNoAllocScratchBytes) return SSM_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != SSM_OK) return st;
  a.cu_seqlens = nullptr;
  a.nseq = int(p->batch);
  return run_scan(a, pl, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, p->discretization == SSM_DISC_ZOH,
                  scratch, kNoAllocScratchBytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_scan_fwd(const ssm_scan_params *p, void *workspace, size_t workspace_bytes,
                          ssm_stream_t stream) {
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, false, a, vec);
  if (st != SSM_OK) return st;
  if (p->batch == 0) return SSM_OK;
  if (p->batch > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  Plan pl;
  if (!make_plan(p, p->batch, false, vec, pl)) return SSM_ERR_UNSUPPORTED;
  a.cu_seqlens = nullptr;
  a.nseq = int(p->batch);
  return run_scan(a, pl, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, p->discretization == SSM_DISC_ZOH,
                  workspace, workspace_bytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_scan_fwd_varlen(const ssm_scan_params *p, const int32_t *cu_seqlens, int64_t nseq,
                                 void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  if (!cu_seqlens || nseq < 0) return SSM_ERR_INVALID_ARG;
  if (nseq > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  if (p && p->seqlen > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;  // int32 offsets
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, true, a, vec);
  if (st != SSM_OK) return st;
  if (nseq == 0) return SSM_OK;
  Plan pl;
  if (!make_plan(p, nseq, true, vec, pl)) return SSM_ERR_UNSUPPORTED;
  a.cu_seqlens = cu_seqlens;
  a.nseq = int(nseq);
  return run_scan(a, pl, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, p->discretization == SSM_DISC_ZOH,
                  workspace, workspace_bytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_scan_fwd_varlen_pool(const ssm_scan_params *p, const int32_t *cu_seqlens, int64_t nseq,
                                      float *pool, int64_t num_slots, const int32_t *slot_ids,
                                      void *workspace, size_t workspace_bytes, ssm_stream_t stream) {
  if (!p || !cu_seqlens || !pool || !slot_ids || nseq < 0 || num_slots <= 0) return SSM_ERR_INVALID_ARG;
  if (p->h0 || p->h_last) return SSM_ERR_INVALID_ARG;  // the pool holds both
  if (nseq > (int64_t(1) << 30)) return SSM_ERR_UNSUPPORTED;
  if (p->seqlen > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;  // int32 offsets
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, true, a, vec);
  if (st != SSM_OK) return st;
  if (nseq == 0) return SSM_OK;
  Plan pl;
  if (!make_plan(p, nseq, true, vec, pl)) return SSM_ERR_UNSUPPORTED;
  a.cu_seqlens = cu_seqlens;
  a.nseq = int(nseq);
  a.h0 = pool;
  a.h_last = pool;
  a.state_slots = slot_ids;
  a.num_slots = num_slots;
  return run_scan(a, pl, p->dtype, p->y_fp32 != 0, int(p->dstate), vec, p->discretization == SSM_DISC_ZOH,
                  workspace, workspace_bytes,
                  reinterpret_cast<cudaStream_t>(stream));
}

ssm_status_t ssm_state_update(float *pool, int64_t num_slots, const int32_t *slot_ids, int64_t R,
                              const ssm_scan_params *p, ssm_stream_t stream) {
  if (!p || !pool || !slot_ids || num_slots <= 0 || R < 0) return SSM_ERR_INVALID_ARG;
  if (p->dtype != SSM_F32 && p->dtype != SSM_BF16) return SSM_ERR_INVALID_ARG;
  if (p->batch != R || p->seqlen != 1 || p->dim <= 0 || p->dstate <= 0) return SSM_ERR_INVALID_ARG;
  if (p->discretization != SSM_DISC_EULER && p->discretization != SSM_DISC_ZOH) return SSM_ERR_INVALID_ARG;
  if (p->ngroups > 1) return SSM_ERR_UNSUPPORTED;  // decode takes one B, C per request
  if (!p->u || !p->delta || !p->B || !p->C || !p->A || !p->y) return SSM_ERR_INVALID_ARG;
  const int64_t N = p->dstate;
  if (N % 4 != 0 || N > ssm::kUpdateMaxState) return SSM_ERR_UNSUPPORTED;
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
  // states per thread: 16 when they divide dstate, else 8, else 4
  const int G = N % 16 == 0 ? 16 : (N % 8 == 0 ? 8 : 4);
  a.tpc = int(N / G);
  const int64_t cpb = ssm::kUpdateThreads / a.tpc;  // channels per block
  const int64_t gx = (p->dim + cpb - 1) / cpb;
  if (gx > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  const dim3 blocks(unsigned(gx), unsigned(R < 65535 ? R : 65535));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool has_z = p->z != nullptr, zoh = p->discretization == SSM_DISC_ZOH;
  using bf16 = __nv_bfloat16;
  ssm_status_t ls;
  if (p->dtype == SSM_BF16 && !p->y_fp32) ls = launch_update<bf16, bf16>(a, G, has_z, zoh, blocks, st);
  else if (p->dtype == SSM_BF16) ls = launch_update<bf16, float>(a, G, has_z, zoh, blocks, st);
  else ls = launch_update<float, float>(a, G, has_z, zoh, blocks, st);
  if (ls != SSM_OK) return ls;
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

ssm_status_t ssm_scan_bwd(const ssm_scan_params *p, const ssm_scan_grads *g, void *workspace,
                          size_t workspace_bytes, ssm_stream_t stream) {
  ScanArgs a;
  bool vec = false;
  ssm_status_t st = prepare_scan(p, false, a, vec, false);
  if (st != SSM_OK) return st;
  if (!g || !g->dy || !g->du || !g->ddelta || !g->dB || !g->dC || !g->dA) return SSM_ERR_INVALID_ARG;
  if (p->z && !g->dz) return SSM_ERR_INVALID_ARG;
  const bool aligned = aligned16(g->dy) && aligned16(g->du) && aligned16(g->ddelta) && (!p->z || aligned16(g->dz));
  BwdPlan bp;
  if (!aligned || !make_bwd_plan(p, vec, bp)) return SSM_ERR_UNSUPPORTED;
  if (p->batch > (int64_t(1) << 30) || bp.nunits > 0x7fffffffLL) return SSM_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < bp.bytes || !aligned16(workspace)) return SSM_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  unsigned char *ws = static_cast<unsigned char *>(workspace);
  const size_t nd = size_t(p->dim);
  if (cudaMemsetAsync(ws, 0, 32, cs) != cudaSuccess ||
      cudaMemsetAsync(g->dA, 0, nd * p->dstate * sizeof(float), cs) != cudaSuccess ||
      (g->dDskip && cudaMemsetAsync(g->dDskip, 0, nd * sizeof(float), cs) != cudaSuccess) ||
      (g->ddelta_bias && cudaMemsetAsync(g->ddelta_bias, 0, nd * sizeof(float), cs) != cudaSuccess))
    return SSM_ERR_CUDA;
  if (p->batch == 0) return SSM_OK;
  if (p->seqlen == 0) {  // nothing to walk: dh0 = dh_last, dB, dC empty
    if (g->dh0) {
      const size_t nb = size_t(p->batch) * nd * p->dstate * sizeof(float);
      if ((g->dh_last ? cudaMemcpyAsync(g->dh0, g->dh_last, nb, cudaMemcpyDeviceToDevice, cs)
                      : cudaMemsetAsync(g->dh0, 0, nb, cs)) != cudaSuccess)
        return SSM_ERR_CUDA;
    }
    return SSM_OK;
  }
  const size_t nbc = size_t(p->batch) * p->dstate * p->seqlen * sizeof(float);
  if (cudaMemsetAsync(g->dB, 0, nbc, cs) != cudaSuccess || cudaMemsetAsync(g->dC, 0, nbc, cs) != cudaSuccess)
    return SSM_ERR_CUDA;
  ssm::BwdArgs bwa{};
  bwa.dy = g->dy; bwa.dh_last = g->dh_last;
  bwa.du = g->du; bwa.ddelta = g->ddelta; bwa.dz = g->dz;
  bwa.dA = g->dA; bwa.dDskip = p->Dskip ? g->dDskip : nullptr; bwa.dbias = p->delta_bias ? g->ddelta_bias : nullptr;
  bwa.dh0 = g->dh0;
  bwa.dB = g->dB; bwa.dC = g->dC;
  bwa.ckpt = reinterpret_cast<float *>(ws + bp.off_ckpt);
  bwa.cumd = reinterpret_cast<float *>(ws + bp.off_cumd);
  bwa.seg_sum = reinterpret_cast<float *>(ws + bp.off_ssum);
  bwa.seg_h = reinterpret_cast<float *>(ws + bp.off_sh);
  bwa.seg_g = reinterpret_cast<float *>(ws + bp.off_sg);
  bwa.nblk = bp.nblk;
  bwa.seg_len = bp.seg_len;
  bwa.nseg = int(bp.nseg);
  bwa.vec_dbc = (aligned16(g->dB) && aligned16(g->dC) && p->seqlen % 4 == 0) ? 1 : 0;
  a.cu_seqlens = nullptr;
  using bf16 = __nv_bfloat16;
  const bool has_z = p->z != nullptr, zoh = p->discretization == SSM_DISC_ZOH;
  auto go = [&](auto t_tag, auto tg_tag) -> ssm_status_t {
    using T = typename decltype(t_tag)::type;
    using TG = typename decltype(tg_tag)::type;
    if (zoh)
      return has_z ? launch_bwd<T, TG, true, true>(a, bwa, bp, p, ws, cs) : launch_bwd<T, TG, false, true>(a, bwa, bp, p, ws, cs);
    return has_z ? launch_bwd<T, TG, true, false>(a, bwa, bp, p, ws, cs) : launch_bwd<T, TG, false, false>(a, bwa, bp, p, ws, cs);
  };
  if (p->dtype == SSM_BF16 && !p->y_fp32) return go(TypeTag<bf16>{}, TypeTag<bf16>{});
  if (p->dtype == SSM_BF16) return go(TypeTag<bf16>{}, TypeTag<float>{});
  return go(TypeTag<float>{}, TypeTag<float>{});
}

ssm_status_t ssm_ssd_fwd(const ssm_ssd_params *p, ssm_stream_t stream) {
  if (!p || !p->x || !p->dt || !p->A || !p->B || !p->C || !p->y) return SSM_ERR_INVALID_ARG;
  if (p->batch < 0 || p->nheads <= 0 || p->headdim <= 0 || p->dstate <= 0 || p->seqlen < 0) return SSM_ERR_INVALID_ARG;
  if (p->headdim != ssm::kSsdP || p->dstate != ssm::kSsdN || p->seqlen % 8 != 0) return SSM_ERR_UNSUPPORTED;
  if (!aligned16(p->x) || !aligned16(p->B) || !aligned16(p->C)) return SSM_ERR_UNSUPPORTED;
  if (p->batch * p->nheads > 0x7fffffffLL || p->seqlen > (int64_t(1) << 40)) return SSM_ERR_UNSUPPORTED;
  if (p->batch == 0 || p->seqlen == 0) {
    if (p->h_last && p->batch > 0) {
      const size_t nb = size_t(p->batch) * p->nheads * p->headdim * p->dstate * sizeof(float);
      cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
      if ((p->h0 ? cudaMemcpyAsync(p->h_last, p->h0, nb, cudaMemcpyDeviceToDevice, cs)
                 : cudaMemsetAsync(p->h_last, 0, nb, cs)) != cudaSuccess)
        return SSM_ERR_CUDA;
    }
    return SSM_OK;
  }
  LaunchInfo li;
  if (launch_info(reinterpret_cast<const void *>(ssm::ssd_chunk_kernel), ssm::kSsdThreads, ssm::kSsdSmemBytes, li) != SSM_OK)
    return SSM_ERR_CUDA;
  ssm::SsdArgs a{};
  a.x = static_cast<const __nv_bfloat16 *>(p->x);
  a.dt = p->dt;
  a.A = p->A;
  a.B = static_cast<const __nv_bfloat16 *>(p->B);
  a.C = static_cast<const __nv_bfloat16 *>(p->C);
  a.h0 = p->h0;
  a.y = static_cast<__nv_bfloat16 *>(p->y);
  a.h_last = p->h_last;
  a.nheads = p->nheads;
  a.seqlen = p->seqlen;
  ssm::ssd_chunk_kernel<<<unsigned(p->batch * p->nheads), ssm::kSsdThreads, ssm::kSsdSmemBytes,
                          reinterpret_cast<cudaStream_t>(stream)>>>(a);
  return cudaGetLastError() == cudaSuccess ? SSM_OK : SSM_ERR_CUDA;
}

#ifdef SSM_TRACE_CTA
// Diagnostic build only: copy the CTA trace of the chunked scan kernel (entries of SM id, start
// and end in global-timer nanoseconds) to `host` and clear it; returns the entry count.
int64_t ssm_debug_read_trace(unsigned long long *host, int64_t max_entries) {
  unsigned int n = 0;
  if (cudaDeviceSynchronize() != cudaSuccess || cudaMemcpyFromSymbol(&n, ssm::g_trace_n, sizeof(n)) != cudaSuccess)
    return -1;
  const int64_t m = std::min<int64_t>(std::min<int64_t>(n, ssm::kTraceMax), max_entries);
  if (m > 0 && cudaMemcpyFromSymbol(host, ssm::g_trace, size_t(m) * 3 * sizeof(unsigned long long)) != cudaSuccess)
    return -1;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(ssm::g_trace_n, &zero, sizeof(zero)) != cudaSuccess) return -1;
  return m;
}
#endif

size_t ssm_scan_bwd_workspace_size(const ssm_scan_params *p) {
  ScanArgs a;
  bool vec = false;
  if (prepare_scan(p, false, a, vec, false) != SSM_OK) return 0;
  BwdPlan bp;
  if (!make_bwd_plan(p, vec, bp)) return 0;
  return bp.bytes;
}

size_t ssm_scan_workspace_size(const ssm_scan_params *p, int64_t nseq) {
  ScanArgs a;
  bool vec = false;
  const bool varlen = nseq > 0;
  if (prepare_scan(p, varlen, a, vec) != SSM_OK) return 0;
  Plan pl;
  if (!make_plan(p, varlen ? nseq : p->batch, varlen, vec, pl)) return 0;
  return pl.ws_bytes;
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

void ssm_test_drop_first_handoff(void) { g_test_drop_first_handoff.store(true); }

}  // extern "C"
