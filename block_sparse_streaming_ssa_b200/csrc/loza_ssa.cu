// loza_ssa.cu -- the C ABI declared in include/loza_ssa.h: argument checks,
// TMA tensor maps, and stream-ordered launches of the sm_100a kernels.
// The library allocates no device memory and never synchronises the device
// (except inside loza_ssa_get_last_device_status, whose job that is).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/loza_ssa.h"
#include "backward.cuh"
#include "decode.cuh"
#include "decode_long.cuh"
#include "prefill.cuh"
#include "schedule.cuh"

namespace {

constexpr int kVersion = 10000;  // 1.0.0
constexpr int kMaxVarlenSeqs = 4000;
// The packed prefill keeps a prefix per sequence in shared memory; beside the
// d_qk = 192 rings that leaves room for this many sequences.
constexpr int kMaxVarlenSeqsDqk192 = 3000;
static_assert(kMaxVarlenSeqsDqk192 + 1 <= loza::PrefillLayout<192, 128>::MAX_PREFIX, "smem");
static_assert(kMaxVarlenSeqs + 1 <= loza::PrefillLayout<128, 128>::MAX_PREFIX, "smem");
constexpr int kMaxDecodeWindow = 4096;
constexpr int kMaxDevices = 64;

thread_local char g_last_error[256] = "";

int cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
  return LOZA_SSA_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
};
DeviceInfo g_dev[kMaxDevices];

// Current device, its SM count, and a one-time check that it is sm_100.
int device_info(DeviceInfo& out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_error, sizeof g_last_error, "device ordinal %d unsupported", dev);
    return LOZA_SSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return cuda_fail(e == cudaSuccess ? cudaErrorSymbolNotFound : e,
                         "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.ready = true;
  }
  if (d.cc_major != 10 || d.cc_minor != 0) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "libloza_ssa is built for sm_100a; device %d is sm_%d%d", dev, d.cc_major,
                  d.cc_minor);
    return LOZA_SSA_ERR_CUDA;
  }
  out = d;
  return LOZA_SSA_OK;
}

// 16-bit tensor map: dims {d0 (innermost), d1, d2}, box {64, box_rows, 1}, 128B swizzle.
int make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, int rank,
             CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
             cuuint32_t box_rows = 128) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, dtype, (cuuint32_t)rank,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return LOZA_SSA_ERR_CUDA;
  }
  return LOZA_SSA_OK;
}

// FP8 latent cache [rows, 576] e4m3: 64-byte boxes of 128 rows, unswizzled
// (the kernel expands them to the bf16 swizzled layout itself).
int make_map_kv8(CUtensorMap* map, const void* base, uint64_t rows) {
  cuuint64_t dims[2] = {(cuuint64_t)loza::kDecodeDqk, rows};
  cuuint64_t strides[1] = {(cuuint64_t)loza::kDecodeDqk};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_error, sizeof g_last_error, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return LOZA_SSA_ERR_CUDA;
  }
  return LOZA_SSA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Dense inputs get their exact work-item count here; packed inputs count
// theirs on the device (items_upper bounds the grid).
template <int DQK, int DV>
int launch_prefill(const void* q, const void* k, const void* v, loza::PrefillParams prm,
                   uint64_t plane_rows, uint64_t planes, long long items_upper, int n_prefix,
                   cudaStream_t stream, const DeviceInfo& dev) {
  using Lay = loza::PrefillLayout<DQK, DV>;
  CUtensorMap mq, mk, mv, mo;
  int rc;
  if ((rc = make_map(&mq, q, DQK, plane_rows, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mk, k, DQK, plane_rows, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mv, v, DV, plane_rows, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mo, prm.o, DV, plane_rows, planes, 3)) != LOZA_SSA_OK) return rc;
  if (prm.cu_seqlens == nullptr) {
    const long long nb = (prm.L + 127) / 128;
    items_upper = (long long)planes * nb;
    prm.total_items = (int)items_upper;
  }
  const size_t smem = Lay::smem_bytes(n_prefix);
  const size_t smem_max = Lay::smem_bytes((DQK == 192 ? kMaxVarlenSeqsDqk192 : kMaxVarlenSeqs) + 1);
  void (*kern)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, loza::PrefillParams) =
      loza::ssa_prefill_kernel<DQK, DV>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill)");
  const int grid = items_upper < dev.num_sms ? (int)items_upper : dev.num_sms;
  if (grid < 1) return LOZA_SSA_OK;
  kern<<<grid, Lay::THREADS, smem, stream>>>(mq, mk, mv, mo, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "prefill launch");
  return LOZA_SSA_OK;
}

int dispatch_prefill(int d_qk, int d_v, const void* q, const void* k, const void* v,
                     const loza::PrefillParams& prm, uint64_t plane_rows, uint64_t planes,
                     long long items_upper, int n_prefix, cudaStream_t s, const DeviceInfo& dev) {
  if (d_qk == 64 && d_v == 64)
    return launch_prefill<64, 64>(q, k, v, prm, plane_rows, planes, items_upper, n_prefix, s,
                                  dev);
  if (d_qk == 128 && d_v == 128)
    return launch_prefill<128, 128>(q, k, v, prm, plane_rows, planes, items_upper, n_prefix, s,
                                    dev);
  if (d_qk == 192 && d_v == 128)
    return launch_prefill<192, 128>(q, k, v, prm, plane_rows, planes, items_upper, n_prefix, s,
                                    dev);
  return LOZA_SSA_ERR_HEAD_DIM;
}

// Backward workspace: D_i (fp32 per row, 256-byte aligned), then the sink
// blocks' fp32 partial dK / dV.
struct BwdWorkspace {
  size_t d_bytes, part_bytes;
};
BwdWorkspace bwd_workspace(long long planes, int L, int d_qk, int d_v, int n_sink) {
  const int nb = (L + 127) / 128;
  const long long rows = planes * L;
  BwdWorkspace w;
  w.d_bytes = (size_t)(((rows * 4) + 255) / 256) * 256;
  w.part_bytes = (size_t)planes * loza::bwd_sink_items(n_sink, nb) * 128 * (d_qk + d_v) * 4;
  return w;
}

bool bwd_dims_ok(int d_qk, int d_v) {
  return (d_qk == 64 && d_v == 64) || (d_qk == 128 && d_v == 128) || (d_qk == 192 && d_v == 128);
}

// q_items / kv_items: the work-item counts (dense) or upper bounds on them
// (packed: the kernels read the exact counts from the prefixes).
template <int DQK, int DV>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
               loza::BwdParams prm, long long q_items, long long kv_items, cudaStream_t s,
               const DeviceInfo& dev) {
  // 128-row boxes for the dQ kernel and for K, V; the dK/dV kernel reads Q and
  // dO in half-steps of 64 rows
  CUtensorMap mq, mk, mv, mdo, mq64, mdo64;
  int rc;
  const uint64_t L = (uint64_t)prm.plane_rows, planes = (uint64_t)prm.planes;
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  if ((rc = make_map(&mq, q, DQK, L, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mk, k, DQK, L, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mv, v, DV, L, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mdo, dout, DV, L, planes, 3)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mq64, q, DQK, L, planes, 3, bf, 64)) != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mdo64, dout, DV, L, planes, 3, bf, 64)) != LOZA_SSA_OK) return rc;
  const long long rows = (long long)prm.planes * prm.plane_rows;
  const int pre_grid = (int)std::min<long long>((rows + 63) / 64, (long long)dev.num_sms * 16);
  loza::ssa_bwd_preprocess_kernel<DV><<<pre_grid, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout),
      const_cast<float*>(prm.dsum), rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "backward preprocess launch");

  using LQ = loza::BwdDqLayout<DQK, DV>;
  if ((e = cudaFuncSetAttribute(loza::ssa_bwd_dq_kernel<DQK, DV>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, LQ::SMEM_BYTES)) !=
      cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(backward dq)");
  if (q_items > 0)
    loza::ssa_bwd_dq_kernel<DQK, DV><<<(int)std::min<long long>(q_items, dev.num_sms),
                                       loza::kBwdThreads, LQ::SMEM_BYTES, s>>>(mq, mk, mv, mdo,
                                                                              prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward dq launch");

  using LK = loza::BwdKvLayout<DQK, DV>;
  if ((e = cudaFuncSetAttribute(loza::ssa_bwd_dkdv_kernel<DQK, DV>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, LK::SMEM_BYTES)) !=
      cudaSuccess)
    return cuda_fail(e, "cudaFuncSetAttribute(backward dkdv)");
  if (kv_items > 0)
    loza::ssa_bwd_dkdv_kernel<DQK, DV><<<(int)std::min<long long>(kv_items, dev.num_sms),
                                         loza::kBwdThreads, LK::SMEM_BYTES, s>>>(
        mq64, mk, mv, mdo64, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward dkdv launch");

  if (prm.cu_seqlens == nullptr && prm.sink_items > 0) {
    const long long quads =
        (long long)prm.planes * std::min(prm.n_sink, prm.nb) * 128 * ((DQK + DV) / 4);
    const int red_grid = (int)std::min<long long>((quads + 255) / 256, (long long)dev.num_sms * 8);
    loza::ssa_bwd_sink_reduce_kernel<DQK, DV><<<red_grid, 256, 0, s>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward reduce launch");
  } else if (prm.cu_seqlens != nullptr && prm.n_sink > 0) {
    // one column of CTAs per sequence; each walks its (head, sink block, row, 4 columns)
    loza::ssa_bwd_sink_reduce_kernel<DQK, DV><<<dim3(8, prm.n_seqs), 256, 0, s>>>(prm);
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "backward reduce launch");
  }
  return LOZA_SSA_OK;
}

int dispatch_bwd(int d_qk, const void* q, const void* k, const void* v, const void* o,
                 const void* dout, const loza::BwdParams& prm, long long q_items,
                 long long kv_items, cudaStream_t s, const DeviceInfo& dev) {
  if (d_qk == 64) return launch_bwd<64, 64>(q, k, v, o, dout, prm, q_items, kv_items, s, dev);
  if (d_qk == 128) return launch_bwd<128, 128>(q, k, v, o, dout, prm, q_items, kv_items, s, dev);
  return launch_bwd<192, 128>(q, k, v, o, dout, prm, q_items, kv_items, s, dev);
}

bool prefill_dims_ok(int d_qk, int d_v) {
  return (d_qk == 64 && d_v == 64) || (d_qk == 128 && d_v == 128) || (d_qk == 192 && d_v == 128);
}

__global__ void debug_tiles_kernel(int n_qb, int n_sink, int n_local, int* tiles, int* counts,
                                   int max_tiles) {
  const int qb = blockIdx.x * blockDim.x + threadIdx.x;
  if (qb >= n_qb) return;
  const loza::TileRange r = loza::tile_range(qb, n_sink, n_local);
  counts[qb] = r.count;
  for (int t = 0; t < r.count && t < max_tiles; ++t)
    tiles[(size_t)qb * max_tiles + t] = loza::tile_block(r, t);
}

__global__ void debug_decode_pages_kernel(loza::DecodeParams p, int* pages, int* counts,
                                          int max_tiles) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= p.B) return;
  loza::DecodeWindow w;
  if (!loza::decode_window(p, b, w)) {
    counts[b] = 0;
    atomicOr(&loza::g_loza_status, LOZA_SSA_DEV_BAD_SEQLEN);
    return;
  }
  counts[b] = w.tr.count;
  for (int i = 0; i < w.tr.count && i < max_tiles; ++i) {
    const int phys = loza::decode_page(p, b, loza::tile_block(w.tr, i));
    if (phys < 0) atomicOr(&loza::g_loza_status, LOZA_SSA_DEV_BAD_PAGE);
    pages[(size_t)b * max_tiles + i] = phys;
  }
}

// One warp; thread 0 waits on an mbarrier that nothing arrives on, through
// the pipelines' bounded wait with a limit of timeout_ns, then the other 31
// threads wait on it too and must give up on the abort flag thread 0 set.
// result[0] = 1 if thread 0's wait gave up, result[1] = how many of the
// others' waits gave up.
__global__ void debug_wait_timeout_kernel(unsigned long long timeout_ns, int* result) {
  __shared__ __align__(8) unsigned long long bar_storage;
  __shared__ int abort_storage;
  const uint32_t bar = loza::smem_u32(&bar_storage);
  volatile int* abort_flag = &abort_storage;
  if (threadIdx.x == 0) {
    loza::mbar_init(bar, 1);
    *abort_flag = 0;
    loza::fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = loza::mbar_wait_for(bar, 0, abort_flag, &loza::g_loza_status,
                                        LOZA_SSA_DEV_WAIT_TIMEOUT, timeout_ns);
    result[0] = ok ? 0 : 1;
  }
  __syncthreads();
  if (threadIdx.x > 0) {
    // ten times the limit, so that only the abort flag ends these waits in time
    const bool ok = loza::mbar_wait_for(bar, 0, abort_flag, &loza::g_loza_status,
                                        LOZA_SSA_DEV_WAIT_TIMEOUT, 10 * timeout_ns);
    const unsigned gave_up = __ballot_sync(0xfffffffeu, !ok);
    if (threadIdx.x == 1) result[1] = __popc(gave_up);
  }
}

// Scratch for loza_ssa_decode_static_scratch: the decode workspace of up to
// LOZA_SSA_STATIC_SCRATCH_SLOTS split slots (fp16 partial O, 256-byte aligned,
// then fp32 partial LSE), resident on every device that loads the library.
// In host code the name only stands for the array; the kernels get its device
// address, looked up once per device.
static __device__ __align__(256) unsigned char g_decode_scratch[LOZA_SSA_STATIC_SCRATCH_BYTES];
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_decode_scratch on the current device (looked up on the
// first call for that device, with the device current).
int static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_error, sizeof g_last_error, "device ordinal %d unsupported", dev);
    return LOZA_SSA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (e != cudaSuccess || !ptr) return cuda_fail(e, "cudaGetSymbolAddress(decode scratch)");
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return LOZA_SSA_OK;
}

// Largest cluster the decode split kernel is launched as: the in-kernel merge
// takes up to 4 splits (8-CTA clusters of this kernel measured much slower
// than the merge kernel: they schedule as fewer, later waves).
constexpr int kMaxClusterSplits = loza::kClusterMergeMaxSplits;

int dev_index() {
  int dev = 0;
  return cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices ? dev : 0;
}

// Whether a cluster of n CTAs of the decode split kernel (its shared memory,
// one CTA per SM) can be resident on the device, asked once per (device,
// kernel, n).
int g_cluster_fit[kMaxDevices][2][kMaxClusterSplits + 1] = {};  // 0 unknown, 1 yes, 2 no

bool cluster_fits(void (*split)(CUtensorMap, CUtensorMap, loza::DecodeParams), int n, int dev) {
  const int kind = split == loza::ssa_decode_split_kernel<true> ? 1 : 0;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_cluster_fit[dev][kind][n]) return g_cluster_fit[dev][kind][n] == 1;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(n, 1, 1);
  cfg.blockDim = dim3(320);
  cfg.dynamicSmemBytes = loza::DecodeLayout::SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = n;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  const cudaError_t e = cudaOccupancyMaxActiveClusters(&clusters, split, &cfg);
  if (e != cudaSuccess) cudaGetLastError();  // not an error of this call: use the merge kernel
  const bool ok = e == cudaSuccess && clusters >= 1;
  std::lock_guard<std::mutex> lock(g_mu);
  g_cluster_fit[dev][kind][n] = ok ? 1 : 2;
  return ok;
}

// Split CTAs per (sequence, head group): listed pages taken two at a time.
int decode_splits(int n_sink, int n_local, int max_extra = 0) {
  return (n_sink + n_local + max_extra + loza::kDecodePagesPerSplit - 1) /
         loza::kDecodePagesPerSplit;
}

size_t decode_partial_floats(int B, int H_q, int n_split) {
  const size_t hg = (size_t)(H_q + 127) / 128;
  return (size_t)B * hg * (size_t)n_split * 128;
}

// Whether a decode of B rows over a window listing n_sink + n_local pages
// and up to max_extra chosen ones takes the long-window kernel (bf16 cache
// only): more than kLongMinPages listed pages, and page offsets that fit in
// int.
bool decode_long_eligible(int B, int H_q, int n_sink, int n_local, int max_extra) {
  const long long units = (long long)B * ((H_q + 127) / 128);
  const long long listed = (long long)n_sink + n_local + max_extra;
  return listed > loza::kLongMinPages && units <= (1ll << 20) && units * listed < (1ll << 31);
}

// Workspace of the long-window kernel: a partial O (fp16) and LSE per slot --
// a unit has one slot per CTA pair its pages span, B * HG + pairs - 1 in all
// -- and the plan's B * HG + 1 page offsets and B * HG (first slot, count)
// pairs.
struct LongWorkspace {
  size_t o, lse, plan, total;
};
LongWorkspace long_workspace(int B, int H_q) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  const size_t units = (size_t)B * ((H_q + 127) / 128);
  const size_t slots = units + loza::kLongMaxPairs;
  LongWorkspace w;
  w.o = 0;
  w.lse = up(slots * 128 * loza::kDecodeDv * sizeof(__half));
  w.plan = w.lse + up(slots * 128 * sizeof(float));
  w.total = w.plan + up((3 * units + 1) * sizeof(int));
  return w;
}

// Workspace of the split kernel: a partial O (fp16) and LSE per split CTA.
size_t decode_split_workspace_size(int B, int H_q, int n_sink, int n_local, int max_extra) {
  const size_t rows = decode_partial_floats(B, H_q, decode_splits(n_sink, n_local, max_extra));
  const size_t o_bytes = rows * loza::kDecodeDv * sizeof(__half);  // partial O is fp16
  const size_t lse_bytes = rows * sizeof(float);
  return ((o_bytes + 255) / 256) * 256 + ((lse_bytes + 255) / 256) * 256;
}

}  // namespace

namespace {

// Device staging of loza_ssa_prefill_host: q, k, v, o and lse, each 256-byte aligned.
struct HostStaging {
  size_t q, k, v, o, lse, total;
};

HostStaging host_staging(long long planes, int L, int d_qk, int d_v) {
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  HostStaging st;
  st.q = up((size_t)planes * L * d_qk * 2);
  st.k = st.q;
  st.v = up((size_t)planes * L * d_v * 2);
  st.o = st.v;
  st.lse = up((size_t)planes * L * 4);
  st.total = st.q + st.k + st.v + st.o + st.lse;
  return st;
}

// Copy streams of the host-buffer call, one pair per device, created once.
cudaStream_t g_h2d[kMaxDevices] = {};
cudaStream_t g_d2h[kMaxDevices] = {};

int copy_streams(cudaStream_t* h2d, cudaStream_t* d2h) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return LOZA_SSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_h2d[dev]) {
    // both streams or neither: a half-made pair is released, not kept
    cudaStream_t up = nullptr, down = nullptr;
    if ((e = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags(h2d)");
    if ((e = cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking)) != cudaSuccess) {
      cudaStreamDestroy(up);
      return cuda_fail(e, "cudaStreamCreateWithFlags(d2h)");
    }
    g_d2h[dev] = down;
    g_h2d[dev] = up;
  }
  *h2d = g_h2d[dev];
  *d2h = g_d2h[dev];
  return LOZA_SSA_OK;
}

// Events of one host-buffer call: created per call, released by the driver
// once the work that records them has completed.
struct EventSet {
  std::vector<cudaEvent_t> ev;
  ~EventSet() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
  }
  cudaError_t make(cudaEvent_t* out) {
    cudaError_t e = cudaEventCreateWithFlags(out, cudaEventDisableTiming);
    if (e == cudaSuccess) ev.push_back(*out);
    return e;
  }
};

}  // namespace

extern "C" {

int loza_ssa_version(void) { return kVersion; }

const char* loza_ssa_last_error_string(void) { return g_last_error; }

const char* loza_ssa_status_string(int status) {
  switch (status) {
    case LOZA_SSA_OK: return "ok";
    case LOZA_SSA_ERR_NULL: return "a required pointer is NULL";
    case LOZA_SSA_ERR_SHAPE: return "a size is out of range, or scale is not finite";
    case LOZA_SSA_ERR_HEAD_DIM: return "unsupported (d_qk, d_v)";
    case LOZA_SSA_ERR_BLOCK: return "block / page_size must be 128";
    case LOZA_SSA_ERR_WINDOW: return "n_sink / n_local out of range";
    case LOZA_SSA_ERR_ALIGN:
      return "pointer not aligned (bf16 tensors: 16 B; prefill o and backward dq, dk, dv: 32 B; "
             "lse: 4 B; workspace: 256 B)";
    case LOZA_SSA_ERR_WORKSPACE: return "decode workspace missing or too small";
    case LOZA_SSA_ERR_CUDA: return "CUDA error (see loza_ssa_last_error_string)";
    case LOZA_SSA_ERR_SCRATCH_LIMIT: return "decode needs more split slots than the built-in scratch holds";
    default: return "unknown status";
  }
}

int loza_ssa_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int L, int d_qk, int d_v, int block, int n_sink, int n_local,
                     float scale, loza_ssa_stream_t stream) {
  if (!q || !k || !v || !o || !lse) return LOZA_SSA_ERR_NULL;
  if (B < 1 || H < 1 || L < 1 || !std::isfinite(scale)) return LOZA_SSA_ERR_SHAPE;
  if (!prefill_dims_ok(d_qk, d_v)) return LOZA_SSA_ERR_HEAD_DIM;
  if (block != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 32) || !aligned(lse, 4))
    return LOZA_SSA_ERR_ALIGN;
  const long long nb = (L + 127) / 128;
  const long long items = (long long)B * H * nb;
  if (items >= (1ll << 31) || (long long)B * H >= (1ll << 31)) return LOZA_SSA_ERR_SHAPE;
  DeviceInfo dev;
  int rc = device_info(dev);
  if (rc != LOZA_SSA_OK) return rc;
  loza::PrefillParams prm{};
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.cu_seqlens = nullptr;
  prm.n_seqs = B;
  prm.H = H;
  prm.L = L;
  prm.plane_rows = L;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.total_items = (int)items;
  return dispatch_prefill(d_qk, d_v, q, k, v, prm, (uint64_t)L, (uint64_t)B * H, items, 0,
                          reinterpret_cast<cudaStream_t>(stream), dev);
}

size_t loza_ssa_prefill_host_workspace_size(int B, int H, int L, int d_qk, int d_v) {
  if (B < 1 || H < 1 || L < 1 || !prefill_dims_ok(d_qk, d_v)) return 0;
  return host_staging((long long)B * H, L, d_qk, d_v).total;
}

int loza_ssa_prefill_host(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int H, int L, int d_qk, int d_v, int block, int n_sink,
                          int n_local, float scale, int n_chunks, void* workspace,
                          size_t workspace_bytes, loza_ssa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !workspace) return LOZA_SSA_ERR_NULL;
  if (B < 1 || H < 1 || L < 1 || n_chunks < 1 || !std::isfinite(scale)) return LOZA_SSA_ERR_SHAPE;
  if (!prefill_dims_ok(d_qk, d_v)) return LOZA_SSA_ERR_HEAD_DIM;
  if (block != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  const long long planes = (long long)B * H;
  const HostStaging st = host_staging(planes, L, d_qk, d_v);
  if (workspace_bytes < st.total) return LOZA_SSA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return LOZA_SSA_ERR_ALIGN;
  cudaStream_t h2d, d2h;
  int rc = copy_streams(&h2d, &d2h);
  if (rc != LOZA_SSA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  char* dq = ws;
  char* dk = dq + st.q;
  char* dv = dk + st.k;
  char* dout = dv + st.v;
  char* dlse = dout + st.o;
  const size_t q_plane = (size_t)L * d_qk * 2, v_plane = (size_t)L * d_v * 2,
               l_plane = (size_t)L * 4;
  const long long chunks = n_chunks < planes ? n_chunks : planes;
  EventSet evs;
  cudaEvent_t start, fin;
  cudaError_t e;
  // everything below follows the caller's earlier work on its stream (which
  // may still read this staging from a previous call)
  if ((e = evs.make(&start)) != cudaSuccess || (e = cudaEventRecord(start, s)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(h2d, start, 0)) != cudaSuccess)
    return cuda_fail(e, "host prefill: start");
  for (long long c = 0; c < chunks; ++c) {
    const long long p0 = planes * c / chunks, p1 = planes * (c + 1) / chunks, np = p1 - p0;
    const char* hq = static_cast<const char*>(q) + p0 * q_plane;
    const char* hk = static_cast<const char*>(k) + p0 * q_plane;
    const char* hv = static_cast<const char*>(v) + p0 * v_plane;
    cudaEvent_t in, done;
    if ((e = cudaMemcpyAsync(dq + p0 * q_plane, hq, np * q_plane, cudaMemcpyHostToDevice, h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(dk + p0 * q_plane, hk, np * q_plane, cudaMemcpyHostToDevice, h2d)) !=
            cudaSuccess ||
        (e = cudaMemcpyAsync(dv + p0 * v_plane, hv, np * v_plane, cudaMemcpyHostToDevice, h2d)) !=
            cudaSuccess ||
        (e = evs.make(&in)) != cudaSuccess || (e = cudaEventRecord(in, h2d)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, in, 0)) != cudaSuccess)
      return cuda_fail(e, "host prefill: upload");
    // the chunk's planes are whole (b, h) planes: one dense call over [1, np, L, d]
    rc = loza_ssa_prefill(dq + p0 * q_plane, dk + p0 * q_plane, dv + p0 * v_plane,
                          dout + p0 * v_plane, reinterpret_cast<float*>(dlse + p0 * l_plane), 1,
                          (int)np, L, d_qk, d_v, block, n_sink, n_local, scale, stream);
    if (rc != LOZA_SSA_OK) return rc;
    if ((e = evs.make(&done)) != cudaSuccess || (e = cudaEventRecord(done, s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(d2h, done, 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(static_cast<char*>(o) + p0 * v_plane, dout + p0 * v_plane,
                             np * v_plane, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(reinterpret_cast<char*>(lse) + p0 * l_plane, dlse + p0 * l_plane,
                             np * l_plane, cudaMemcpyDeviceToHost, d2h)) != cudaSuccess)
      return cuda_fail(e, "host prefill: download");
  }
  // the caller's stream completes once the last download has
  if ((e = evs.make(&fin)) != cudaSuccess || (e = cudaEventRecord(fin, d2h)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(s, fin, 0)) != cudaSuccess)
    return cuda_fail(e, "host prefill: finish");
  return LOZA_SSA_OK;
}

size_t loza_ssa_prefill_bwd_workspace_size(int B, int H, int L, int d_qk, int d_v, int n_sink,
                                           int n_local) {
  if (B < 1 || H < 1 || L < 1 || !bwd_dims_ok(d_qk, d_v) || n_sink < 0 || n_local < 1)
    return 0;
  const BwdWorkspace w = bwd_workspace((long long)B * H, L, d_qk, d_v, n_sink);
  return w.d_bytes + w.part_bytes;
}

int loza_ssa_prefill_bwd(const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B,
                         int H, int L, int d_qk, int d_v, int block, int n_sink, int n_local,
                         float scale, void* workspace, size_t workspace_bytes,
                         loza_ssa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return LOZA_SSA_ERR_NULL;
  if (B < 1 || H < 1 || L < 1 || !std::isfinite(scale)) return LOZA_SSA_ERR_SHAPE;
  if (!bwd_dims_ok(d_qk, d_v)) return LOZA_SSA_ERR_HEAD_DIM;
  if (block != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 32) || !aligned(dk, 32) || !aligned(dv, 32) ||
      !aligned(lse, 4))
    return LOZA_SSA_ERR_ALIGN;
  const long long nb = (L + 127) / 128;
  const long long planes = (long long)B * H;
  const long long sink_items = loza::bwd_sink_items(n_sink, (int)std::min<long long>(nb, 1 << 30));
  if (planes * nb >= (1ll << 31) || planes * (sink_items + nb) >= (1ll << 31) ||
      planes * L >= (1ll << 40))
    return LOZA_SSA_ERR_SHAPE;
  const size_t need = loza_ssa_prefill_bwd_workspace_size(B, H, L, d_qk, d_v, n_sink, n_local);
  if (!workspace || workspace_bytes < need) return LOZA_SSA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return LOZA_SSA_ERR_ALIGN;
  DeviceInfo dev;
  int rc = device_info(dev);
  if (rc != LOZA_SSA_OK) return rc;
  const BwdWorkspace w = bwd_workspace(planes, L, d_qk, d_v, n_sink);
  loza::BwdParams prm{};
  prm.lse = lse;
  prm.dsum = reinterpret_cast<const float*>(workspace);
  prm.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + w.d_bytes);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.L = L;
  prm.planes = (int)planes;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.nb = (int)nb;
  prm.sink_items = (int)sink_items;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu_seqlens = nullptr;
  prm.pfx = nullptr;
  prm.n_seqs = B;
  prm.plane_rows = L;
  const long long q_items = planes * nb;
  const long long kv_items = planes * (sink_items + (nb > n_sink ? nb - n_sink : 0));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return dispatch_bwd(d_qk, q, k, v, o, dout, prm, q_items, kv_items, s, dev);
}

// Packed backward workspace: D per row, the three prefixes, then the sink
// partials for an upper bound on the sink slots: sequence s has at most
// n_sink sink blocks of at most ceil(nb_s / 8) chunks, and
// sum_s nb_s <= total / 128 + n_seqs (the bound holds whatever the lengths;
// the setup kernel also refuses a count above it).
struct BwdVarlenWorkspace {
  size_t d_bytes, pfx_bytes, part_bytes;
  long long q_items_upper, kv_items_upper, sink_slots;
};
BwdVarlenWorkspace bwd_varlen_workspace(int n_seqs, int total, int max_seqlen, int H, int d_qk,
                                        int d_v, int n_sink, int n_local) {
  (void)n_local;
  BwdVarlenWorkspace w;
  (void)max_seqlen;
  const long long sum_nb = (long long)total / 128 + n_seqs;
  const long long sink_slots =
      (long long)H * n_sink * ((sum_nb + 7 * (long long)n_seqs) / 8 + n_seqs);
  w.d_bytes = (size_t)((((long long)H * total * 4) + 255) / 256) * 256;
  w.pfx_bytes = (size_t)((3 * ((long long)n_seqs + 1) * 4 + 255) / 256) * 256;
  w.part_bytes = (size_t)sink_slots * 128 * (d_qk + d_v) * 4;
  w.q_items_upper = (long long)H * sum_nb;
  w.kv_items_upper = w.q_items_upper + sink_slots;
  w.sink_slots = sink_slots;
  return w;
}

size_t loza_ssa_prefill_varlen_bwd_workspace_size(int n_seqs, int total_tokens, int max_seqlen,
                                                  int H, int d_qk, int d_v, int n_sink,
                                                  int n_local) {
  if (n_seqs < 1 || n_seqs > kMaxVarlenSeqs || total_tokens < 1 || max_seqlen < 1 || H < 1 ||
      !bwd_dims_ok(d_qk, d_v) || n_sink < 0 || n_local < 1)
    return 0;
  const BwdVarlenWorkspace w =
      bwd_varlen_workspace(n_seqs, total_tokens, max_seqlen, H, d_qk, d_v, n_sink, n_local);
  return w.d_bytes + w.pfx_bytes + w.part_bytes;
}

int loza_ssa_prefill_varlen_bwd(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                const int* cu_seqlens, int n_seqs, int total_tokens,
                                int max_seqlen, int H, int d_qk, int d_v, int block, int n_sink,
                                int n_local, float scale, void* workspace, size_t workspace_bytes,
                                loza_ssa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv || !cu_seqlens)
    return LOZA_SSA_ERR_NULL;
  if (n_seqs < 1 || n_seqs > kMaxVarlenSeqs || total_tokens < 1 || max_seqlen < 1 || H < 1 ||
      !std::isfinite(scale))
    return LOZA_SSA_ERR_SHAPE;
  if (!bwd_dims_ok(d_qk, d_v)) return LOZA_SSA_ERR_HEAD_DIM;
  if (block != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 32) || !aligned(dk, 32) || !aligned(dv, 32) ||
      !aligned(lse, 4) || !aligned(cu_seqlens, 4))
    return LOZA_SSA_ERR_ALIGN;
  const BwdVarlenWorkspace w =
      bwd_varlen_workspace(n_seqs, total_tokens, max_seqlen, H, d_qk, d_v, n_sink, n_local);
  if (w.kv_items_upper >= (1ll << 31)) return LOZA_SSA_ERR_SHAPE;
  const size_t need = w.d_bytes + w.pfx_bytes + w.part_bytes;
  if (!workspace || workspace_bytes < need) return LOZA_SSA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return LOZA_SSA_ERR_ALIGN;
  DeviceInfo dev;
  int rc = device_info(dev);
  if (rc != LOZA_SSA_OK) return rc;
  char* ws = static_cast<char*>(workspace);
  int* pfx = reinterpret_cast<int*>(ws + w.d_bytes);
  loza::BwdParams prm{};
  prm.lse = lse;
  prm.dsum = reinterpret_cast<const float*>(ws);
  prm.part = reinterpret_cast<float*>(ws + w.d_bytes + w.pfx_bytes);
  prm.dq = static_cast<__nv_bfloat16*>(dq);
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.L = max_seqlen;
  prm.planes = H;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.cu_seqlens = cu_seqlens;
  prm.pfx = pfx;
  prm.n_seqs = n_seqs;
  prm.plane_rows = total_tokens;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  loza::ssa_bwd_varlen_setup_kernel<<<1, 1024, 0, s>>>(cu_seqlens, n_seqs, total_tokens, H,
                                                        n_sink, w.sink_slots, pfx);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "backward varlen setup launch");
  return dispatch_bwd(d_qk, q, k, v, o, dout, prm, w.q_items_upper, w.kv_items_upper, s, dev);
}

int loza_ssa_prefill_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                            const int* cu_seqlens, int n_seqs, int total_tokens, int max_seqlen,
                            int H, int d_qk, int d_v, int block, int n_sink, int n_local,
                            float scale, loza_ssa_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !cu_seqlens) return LOZA_SSA_ERR_NULL;
  if (n_seqs < 1 || n_seqs > kMaxVarlenSeqs || total_tokens < 1 || max_seqlen < 1 || H < 1 ||
      !std::isfinite(scale))
    return LOZA_SSA_ERR_SHAPE;
  if (!prefill_dims_ok(d_qk, d_v)) return LOZA_SSA_ERR_HEAD_DIM;
  if (d_qk == 192 && n_seqs > kMaxVarlenSeqsDqk192) return LOZA_SSA_ERR_SHAPE;
  if (block != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 32) ||
      !aligned(lse, 4) || !aligned(cu_seqlens, 4))
    return LOZA_SSA_ERR_ALIGN;
  // sum_s ceil(len_s/128) <= total/128 + n_seqs bounds the work-item count
  const long long upper = (long long)H * ((long long)total_tokens / 128 + n_seqs);
  if (upper >= (1ll << 31)) return LOZA_SSA_ERR_SHAPE;
  DeviceInfo dev;
  int rc = device_info(dev);
  if (rc != LOZA_SSA_OK) return rc;
  loza::PrefillParams prm{};
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.cu_seqlens = cu_seqlens;
  prm.n_seqs = n_seqs;
  prm.H = H;
  prm.L = max_seqlen;
  prm.plane_rows = total_tokens;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.total_items = 0;
  return dispatch_prefill(d_qk, d_v, q, k, v, prm, (uint64_t)total_tokens, (uint64_t)H,
                          upper, n_seqs + 1, reinterpret_cast<cudaStream_t>(stream), dev);
}

size_t loza_ssa_decode_selected_workspace_size(int B, int H_q, int d_v, int n_sink, int n_local,
                                               int max_extra) {
  if (B < 1 || H_q < 1 || d_v != loza::kDecodeDv || n_sink < 0 || n_local < 1 ||
      max_extra < 0 || (long long)n_sink + n_local + max_extra > kMaxDecodeWindow)
    return 0;
  const size_t split = decode_split_workspace_size(B, H_q, n_sink, n_local, max_extra);
  // a long window takes the long-window kernel for a bf16 cache and the split
  // kernel for an FP8 one: room for either
  if (!decode_long_eligible(B, H_q, n_sink, n_local, max_extra)) return split;
  const size_t lng = long_workspace(B, H_q).total;
  return lng > split ? lng : split;
}

size_t loza_ssa_decode_workspace_size(int B, int H_q, int d_v, int n_sink, int n_local) {
  return loza_ssa_decode_selected_workspace_size(B, H_q, d_v, n_sink, n_local, 0);
}

size_t loza_ssa_decode_mtp_workspace_size(int B, int q_len, int H_q, int d_v, int n_sink,
                                          int n_local) {
  if (B < 1 || q_len < 1 || (long long)B * q_len > 65535) return 0;
  return loza_ssa_decode_selected_workspace_size(B * q_len, H_q, d_v, n_sink, n_local, 0);
}

}  // extern "C"

namespace {

// The argument checks of decode_impl up to (not including) the workspace.
int decode_check_args(const void* q, const void* paged_kv, const int* page_table,
                      const int* seq_lens, const int* extra_pages, int max_extra, int q_len,
                      const void* o, const float* lse, int B, int H_q, int d_qk, int d_v,
                      int page_size, int max_pages, int n_pages, int n_sink, int n_local,
                      float scale, const float* kv_scale) {
  if (!q || !paged_kv || !page_table || !seq_lens || !o || !lse) return LOZA_SSA_ERR_NULL;
  if (max_extra < 0 || q_len < 1) return LOZA_SSA_ERR_SHAPE;
  if (q_len > 1 && max_extra > 0) return LOZA_SSA_ERR_SHAPE;  // no public call combines them
  if (B >= 1 && (long long)B * q_len > 65535) return LOZA_SSA_ERR_SHAPE;
  B *= q_len;  // from here on B counts rows: (sequence, query token) pairs
  if (max_extra > 0 && !extra_pages) return LOZA_SSA_ERR_NULL;
  if (max_extra > 0 && !aligned(extra_pages, 4)) return LOZA_SSA_ERR_ALIGN;
  if (B < 1 || H_q < 1 || max_pages < 1 || n_pages < 1 || !std::isfinite(scale))
    return LOZA_SSA_ERR_SHAPE;
  if (B > 65535 || (H_q + 127) / 128 > 65535 || (long long)n_pages * 128 >= (1ll << 31))
    return LOZA_SSA_ERR_SHAPE;
  if (d_qk != loza::kDecodeDqk || d_v != loza::kDecodeDv) return LOZA_SSA_ERR_HEAD_DIM;
  if (page_size != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1 || (long long)n_sink + n_local + max_extra > kMaxDecodeWindow)
    return LOZA_SSA_ERR_WINDOW;
  if (!aligned(q, 16) || !aligned(paged_kv, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(page_table, 4) || !aligned(seq_lens, 4) || !aligned(kv_scale, 4))
    return LOZA_SSA_ERR_ALIGN;
  return LOZA_SSA_OK;
}

// The long-window path: plan kernel, long-window kernel (a programmatic
// dependent of the plan), merge kernel (a programmatic dependent of the long
// kernel).  B counts rows; the arguments are checked.
int decode_long_launch(const void* q, const void* paged_kv, const int* page_table,
                       const int* seq_lens, const int* extra_pages, int max_extra, int q_len,
                       void* o, float* lse, int B, int H_q,
                       int max_pages, int n_pages, int n_sink, int n_local, float scale,
                       void* workspace, const DeviceInfo& dev, cudaStream_t s) {
  const LongWorkspace ws = long_workspace(B, H_q);
  char* base = static_cast<char*>(workspace);
  loza::DecodeParams prm{};
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.o_part = reinterpret_cast<__half*>(base + ws.o);
  prm.lse_part = reinterpret_cast<float*>(base + ws.lse);
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.B = B;
  prm.q_len = q_len;
  prm.H_q = H_q;
  prm.HG = (H_q + 127) / 128;
  prm.max_pages = max_pages;
  prm.n_pages = n_pages;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.n_split = 0;
  prm.extra_pages = max_extra > 0 ? extra_pages : nullptr;
  prm.max_extra = max_extra > 0 ? max_extra : 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wave = INT_MAX;
  int* plan = reinterpret_cast<int*>(base + ws.plan);
  prm.plan = plan;
  prm.n_pairs = std::min(std::max(dev.num_sms / 2, 1), loza::kLongMaxPairs);

  CUtensorMap mq, mkv;
  int rc = make_map(&mq, q, loza::kDecodeDqk, (uint64_t)H_q, (uint64_t)B, 3);
  if (rc != LOZA_SSA_OK) return rc;
  if ((rc = make_map(&mkv, paged_kv, loza::kDecodeDqk, (uint64_t)n_pages * 128, 1, 2)) !=
      LOZA_SSA_OK)
    return rc;
  cudaError_t e = cudaFuncSetAttribute(loza::ssa_decode_long_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       loza::LongDecodeLayout::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode long)");
  loza::ssa_decode_plan_kernel<<<1, loza::kLongPlanThreads, 0, s>>>(prm, plan);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "decode plan launch");
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * prm.n_pairs);
  cfg.blockDim = dim3(loza::LongDecodeLayout::THREADS);
  cfg.dynamicSmemBytes = loza::LongDecodeLayout::SMEM_BYTES;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((e = cudaLaunchKernelEx(&cfg, loza::ssa_decode_long_kernel, mq, mkv, prm)) != cudaSuccess)
    return cuda_fail(e, "decode long launch");
  cfg.gridDim = dim3(B * ((H_q + loza::kMergeHeads - 1) / loza::kMergeHeads));
  cfg.blockDim = dim3(loza::kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  if ((e = cudaLaunchKernelEx(&cfg, loza::ssa_decode_merge_kernel<true>, prm)) != cudaSuccess)
    return cuda_fail(e, "decode merge launch");
  return LOZA_SSA_OK;
}

// loza_ssa_decode with an optional per-sequence list of extra pages
// (extra_pages == nullptr and max_extra == 0: the plain window), q_len
// query tokens per sequence (q_len == 1: one) and an FP8 cache (kv_scale !=
// nullptr: paged_kv holds e4m3 codes).  B counts sequences.
int decode_impl(const void* q, const void* paged_kv, const int* page_table, const int* seq_lens,
                const int* extra_pages, int max_extra, int q_len, void* o, float* lse, int B,
                int H_q, int d_qk, int d_v, int page_size, int max_pages, int n_pages, int n_sink,
                int n_local, float scale, void* workspace, size_t workspace_bytes,
                loza_ssa_stream_t stream, const float* kv_scale = nullptr,
                bool allow_long = true) {
  int rc = decode_check_args(q, paged_kv, page_table, seq_lens, extra_pages, max_extra, q_len, o,
                             lse, B, H_q, d_qk, d_v, page_size, max_pages, n_pages, n_sink,
                             n_local, scale, kv_scale);
  if (rc != LOZA_SSA_OK) return rc;
  B *= q_len;  // from here on B counts rows: (sequence, query token) pairs
  const bool use_long =
      allow_long && !kv_scale && decode_long_eligible(B, H_q, n_sink, n_local, max_extra);
  // what the size query promises (room for either kernel), or, for the
  // built-in scratch (split kernel only), the split kernel's share
  const size_t need =
      allow_long ? loza_ssa_decode_selected_workspace_size(B, H_q, d_v, n_sink, n_local, max_extra)
                 : decode_split_workspace_size(B, H_q, n_sink, n_local, max_extra);
  if (!workspace || workspace_bytes < need) return LOZA_SSA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return LOZA_SSA_ERR_ALIGN;
  DeviceInfo dev;
  rc = device_info(dev);
  if (rc != LOZA_SSA_OK) return rc;
  if (use_long)
    return decode_long_launch(q, paged_kv, page_table, seq_lens, extra_pages, max_extra, q_len, o,
                              lse, B, H_q, max_pages, n_pages, n_sink, n_local, scale, workspace,
                              dev, reinterpret_cast<cudaStream_t>(stream));

  const int n_split = decode_splits(n_sink, n_local, max_extra);
  const int HG = (H_q + 127) / 128;
  const size_t rows = decode_partial_floats(B, H_q, n_split);
  if (rows >= (1ull << 31)) return LOZA_SSA_ERR_SHAPE;  // keeps the CTA index math in int
  loza::DecodeParams prm{};
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.o_part = static_cast<__half*>(workspace);
  prm.lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          ((rows * loza::kDecodeDv * sizeof(__half) + 255) / 256) * 256);
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.B = B;
  prm.q_len = q_len;
  prm.H_q = H_q;
  prm.HG = HG;
  prm.max_pages = max_pages;
  prm.n_pages = n_pages;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  prm.n_split = n_split;
  prm.extra_pages = max_extra > 0 ? extra_pages : nullptr;
  prm.max_extra = max_extra > 0 ? max_extra : 0;
  prm.scale_log2 = scale * 1.4426950408889634f;
  // The split kernel pulls the pages of the CTA one wave later (prm.wave = one
  // CTA per SM) into L2.  In a grid of more than two waves -- a full-attention
  // layer over many pages -- those prefetches evict the current wave's pages
  // before their V columns are read again: measured on the 128K-token
  // full-attention layer, 2.04-2.36 ms without them against 2.56-2.92 ms with.
  // Such grids get no prefetch (the "next wave" index lies past the grid).
  const long long split_ctas = (long long)B * HG * n_split;
  prm.wave = split_ctas <= 2LL * dev.num_sms ? dev.num_sms : INT_MAX;
  prm.kv_scale = kv_scale;

  CUtensorMap mq, mkv;
  if ((rc = make_map(&mq, q, loza::kDecodeDqk, (uint64_t)H_q, (uint64_t)B, 3)) != LOZA_SSA_OK)
    return rc;
  rc = kv_scale ? make_map_kv8(&mkv, paged_kv, (uint64_t)n_pages * 128)
                : make_map(&mkv, paged_kv, loza::kDecodeDqk, (uint64_t)n_pages * 128, 1, 2);
  if (rc != LOZA_SSA_OK) return rc;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void (*split)(CUtensorMap, CUtensorMap, loza::DecodeParams) =
      kv_scale ? loza::ssa_decode_split_kernel<true> : loza::ssa_decode_split_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       loza::DecodeLayout::SMEM_BYTES);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode)");
  dim3 grid(n_split, HG, B);
  // Up to 8 splits per (row, head group): launch them as one cluster, which
  // merges its partials itself (the cluster's CTAs are resident together, so
  // they can wait for each other); more splits (long windows) go through the
  // merge kernel.
  if (n_split <= kMaxClusterSplits && cluster_fits(split, n_split, dev_index())) {
    prm.cluster_merge = 1;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(320);
    cfg.dynamicSmemBytes = loza::DecodeLayout::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = n_split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, split, mq, mkv, prm)) != cudaSuccess)
      return cuda_fail(e, "decode split launch (cluster)");
    return LOZA_SSA_OK;
  }
  prm.cluster_merge = 0;
  split<<<grid, 320, loza::DecodeLayout::SMEM_BYTES, s>>>(mq, mkv, prm);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "decode split launch");
  // the merge is a programmatic dependent of the split kernel: it is scheduled
  // as split CTAs retire and waits (griddepcontrol.wait) for their results
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(B * ((H_q + loza::kMergeHeads - 1) / loza::kMergeHeads));
  cfg.blockDim = dim3(loza::kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if ((e = cudaLaunchKernelEx(&cfg, loza::ssa_decode_merge_kernel<false>, prm)) != cudaSuccess)
    return cuda_fail(e, "decode merge launch");
  return LOZA_SSA_OK;
}

}  // namespace

extern "C" {

int loza_ssa_decode(const void* q, const void* paged_kv, const int* page_table,
                    const int* seq_lens, void* o, float* lse, int B, int H_q, int d_qk, int d_v,
                    int page_size, int max_pages, int n_pages, int n_sink, int n_local,
                    float scale, void* workspace, size_t workspace_bytes,
                    loza_ssa_stream_t stream) {
  return decode_impl(q, paged_kv, page_table, seq_lens, nullptr, 0, 1, o, lse, B, H_q, d_qk,
                     d_v, page_size, max_pages, n_pages, n_sink, n_local, scale, workspace,
                     workspace_bytes, stream);
}

int loza_ssa_decode_mtp(const void* q, const void* paged_kv, const int* page_table,
                        const int* seq_lens, int q_len, void* o, float* lse, int B, int H_q,
                        int d_qk, int d_v, int page_size, int max_pages, int n_pages, int n_sink,
                        int n_local, float scale, void* workspace, size_t workspace_bytes,
                        loza_ssa_stream_t stream) {
  return decode_impl(q, paged_kv, page_table, seq_lens, nullptr, 0, q_len, o, lse, B, H_q, d_qk,
                     d_v, page_size, max_pages, n_pages, n_sink, n_local, scale, workspace,
                     workspace_bytes, stream);
}

int loza_ssa_decode_selected(const void* q, const void* paged_kv, const int* page_table,
                             const int* seq_lens, const int* extra_pages, int max_extra, void* o,
                             float* lse, int B, int H_q, int d_qk, int d_v, int page_size,
                             int max_pages, int n_pages, int n_sink, int n_local, float scale,
                             void* workspace, size_t workspace_bytes,
                             loza_ssa_stream_t stream) {
  return decode_impl(q, paged_kv, page_table, seq_lens, extra_pages, max_extra, 1, o, lse, B,
                     H_q, d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local, scale,
                     workspace, workspace_bytes, stream);
}

int loza_ssa_decode_fp8(const void* q, const void* paged_kv_fp8, const float* kv_scale,
                        const int* page_table, const int* seq_lens, void* o, float* lse, int B,
                        int H_q, int d_qk, int d_v, int page_size, int max_pages, int n_pages,
                        int n_sink, int n_local, float scale, void* workspace,
                        size_t workspace_bytes, loza_ssa_stream_t stream) {
  if (!kv_scale) return LOZA_SSA_ERR_NULL;
  return decode_impl(q, paged_kv_fp8, page_table, seq_lens, nullptr, 0, 1, o, lse, B, H_q, d_qk,
                     d_v, page_size, max_pages, n_pages, n_sink, n_local, scale, workspace,
                     workspace_bytes, stream, kv_scale);
}

size_t loza_ssa_decode_layers_workspace_size(int B, int H_q, int d_v, int max_pages, int n_sink,
                                             int n_local, int any_full) {
  const size_t ssa = loza_ssa_decode_workspace_size(B, H_q, d_v, n_sink, n_local);
  if (!any_full) return ssa;
  const size_t full = loza_ssa_decode_workspace_size(B, H_q, d_v, 0, max_pages);
  if (ssa == 0 || full == 0) return 0;
  return full > ssa ? full : ssa;
}

int loza_ssa_decode_layers(const loza_ssa_decode_layer* layers, int n_layers,
                           const int* page_table, const int* seq_lens, int B, int H_q, int d_qk,
                           int d_v, int page_size, int max_pages, int n_pages, int n_sink,
                           int n_local, float scale, void* workspace, size_t workspace_bytes,
                           loza_ssa_stream_t stream) {
  if (!layers) return LOZA_SSA_ERR_NULL;
  if (n_layers < 1) return LOZA_SSA_ERR_SHAPE;
  for (int i = 0; i < n_layers; ++i) {
    const loza_ssa_decode_layer& l = layers[i];
    // full attention: the window of all max_pages pages ending at the query's
    const int ws = l.full_attention ? 0 : n_sink;
    const int wl = l.full_attention ? max_pages : n_local;
    const int rc = decode_impl(l.q, l.paged_kv, page_table, seq_lens, nullptr, 0, 1, l.o, l.lse,
                               B, H_q, d_qk, d_v, page_size, max_pages, n_pages, ws, wl, scale,
                               workspace, workspace_bytes, stream);
    if (rc != LOZA_SSA_OK) return rc;
  }
  return LOZA_SSA_OK;
}

int loza_ssa_decode_static_scratch(const void* q, const void* paged_kv, const int* page_table,
                                   const int* seq_lens, void* o, float* lse, int B, int H_q,
                                   int d_qk, int d_v, int page_size, int max_pages, int n_pages,
                                   int n_sink, int n_local, float scale,
                                   loza_ssa_stream_t stream) {
  // Same checks and kernels as loza_ssa_decode; only the workspace differs.
  // The argument checks come first, so that a bad call gets the code
  // loza_ssa_decode would give it; the scratch limit only applies to a
  // valid one.
  int rc = decode_check_args(q, paged_kv, page_table, seq_lens, nullptr, 0, 1, o, lse, B, H_q,
                             d_qk, d_v, page_size, max_pages, n_pages, n_sink, n_local, scale,
                             nullptr);
  if (rc != LOZA_SSA_OK) return rc;
  const long long slots = (long long)B * ((H_q + 127) / 128) * decode_splits(n_sink, n_local);
  if (slots > LOZA_SSA_STATIC_SCRATCH_SLOTS) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "decode_static_scratch: B * ceil(H_q/128) * ceil((n_sink + n_local)/2) = %lld split "
                  "slots, the built-in scratch holds %d",
                  slots, LOZA_SSA_STATIC_SCRATCH_SLOTS);
    return LOZA_SSA_ERR_SCRATCH_LIMIT;
  }
  // the built-in scratch is sized for the split kernel, which this call
  // always uses
  const size_t need = decode_split_workspace_size(B, H_q, n_sink, n_local, 0);
  if (need == 0 || need > sizeof(g_decode_scratch)) {
    std::snprintf(g_last_error, sizeof g_last_error,
                  "decode_static_scratch: needs %zu scratch bytes, the built-in scratch holds %zu",
                  need, sizeof(g_decode_scratch));
    return LOZA_SSA_ERR_SCRATCH_LIMIT;
  }
  void* scratch = nullptr;
  if ((rc = static_scratch_address(&scratch)) != LOZA_SSA_OK) return rc;
  return decode_impl(q, paged_kv, page_table, seq_lens, nullptr, 0, 1, o, lse, B, H_q, d_qk, d_v,
                     page_size, max_pages, n_pages, n_sink, n_local, scale, scratch,
                     sizeof(g_decode_scratch), stream, nullptr, /*allow_long=*/false);
}

int loza_ssa_get_last_device_status(loza_ssa_stream_t stream) {
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int v = 0;
  if ((e = cudaMemcpyFromSymbol(&v, loza::g_loza_status, sizeof v)) != cudaSuccess)
    return cuda_fail(e, "read device status");
  const int zero = 0;
  if ((e = cudaMemcpyToSymbol(loza::g_loza_status, &zero, sizeof zero)) != cudaSuccess)
    return cuda_fail(e, "clear device status");
  return v;
}

int loza_ssa_debug_enumerate_tiles(int n_qblocks, int n_sink, int n_local, int* tiles,
                                   int* counts, int max_tiles, loza_ssa_stream_t stream) {
  if (!tiles || !counts) return LOZA_SSA_ERR_NULL;
  if (n_qblocks < 1 || max_tiles < 1) return LOZA_SSA_ERR_SHAPE;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  debug_tiles_kernel<<<(n_qblocks + 127) / 128, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      n_qblocks, n_sink, n_local, tiles, counts, max_tiles);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOZA_SSA_OK : cuda_fail(e, "debug tiles launch");
}

int loza_ssa_debug_wait_timeout(int timeout_us, int* result, loza_ssa_stream_t stream) {
  if (!result) return LOZA_SSA_ERR_NULL;
  if (timeout_us < 1 || timeout_us > 100000) return LOZA_SSA_ERR_SHAPE;
  if (!aligned(result, 4)) return LOZA_SSA_ERR_ALIGN;
  debug_wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      1000ull * (unsigned long long)timeout_us, result);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOZA_SSA_OK : cuda_fail(e, "debug wait-timeout launch");
}

int loza_ssa_debug_long_partition(const int* unit_pages, int n_units, int pairs_launched,
                                  long long* pair_start, int* slot_first, int* slot_count) {
  if (!unit_pages || !pair_start || !slot_first || !slot_count) return LOZA_SSA_ERR_NULL;
  if (n_units < 1 || pairs_launched < 1) return LOZA_SSA_ERR_SHAPE;
  long long T = 0;
  for (int u = 0; u < n_units; ++u) {
    if (unit_pages[u] < 0) return LOZA_SSA_ERR_SHAPE;
    T += unit_pages[u];
  }
  const int P = loza::long_pairs(pairs_launched, T);
  for (int k = 0; k <= pairs_launched; ++k)
    pair_start[k] = k <= P ? loza::long_pair_start(k, T, P) : T;
  long long run = 0;
  for (int u = 0; u < n_units; ++u) {
    loza::long_unit_slot_range(u, run, unit_pages[u], T, P, slot_first + u, slot_count + u);
    run += unit_pages[u];
  }
  return LOZA_SSA_OK;
}

int loza_ssa_debug_decode_pages(const int* page_table, const int* seq_lens, int B, int max_pages,
                                int n_pages, int page_size, int n_sink, int n_local, int* pages,
                                int* counts, int max_tiles, loza_ssa_stream_t stream) {
  if (!page_table || !seq_lens || !pages || !counts) return LOZA_SSA_ERR_NULL;
  if (B < 1 || max_pages < 1 || n_pages < 1 || max_tiles < 1) return LOZA_SSA_ERR_SHAPE;
  if (page_size != 128) return LOZA_SSA_ERR_BLOCK;
  if (n_sink < 0 || n_local < 1) return LOZA_SSA_ERR_WINDOW;
  loza::DecodeParams prm{};
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.B = B;
  prm.q_len = 1;
  prm.max_pages = max_pages;
  prm.n_pages = n_pages;
  prm.n_sink = n_sink;
  prm.n_local = n_local;
  debug_decode_pages_kernel<<<(B + 127) / 128, 128, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      prm, pages, counts, max_tiles);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LOZA_SSA_OK : cuda_fail(e, "debug decode pages launch");
}

}  // extern "C"
