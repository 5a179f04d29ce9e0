// All-gather + rerange in one kernel, push style: each rank stores its own K/V
// rows directly into every rank's paged pool (its own and its peers', the
// peers' pools mapped into this GPU's address space).  The pages
// ("sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// _all_gather_reorganized + materialize_full_kv) all-gather the padded shards
// into one buffer and then scatter that buffer into the pool; here the rows
// cross the link once, straight to their final slots:
//     pool_j[out_cache_loc_j[t]] = local[i]    (t = natural token of local row i)
// for every destination j.  Each 16-byte vector is loaded once and stored
// n_dst times.  Pure data movement: bound by HBM on one GPU and by the NVLink
// bandwidth per GPU when the destinations are peers.
//
// Also the inter-process handle helpers that map a peer's pool.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>
#include <string>

#include "nvtx_range.h"
#include "zz_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ int4 ld_stream(const int4* p) {
  int4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

struct PushArgs {
  const int4* src[2];                      // K, V local rows
  int4* dst[2][ZZ_MAX_PUSH_DST];           // pools per tensor and destination
  const int64_t* loc[ZZ_MAX_PUSH_DST];     // slot map per destination
  const int32_t* tok;                      // local row -> natural token
  int64_t rows;                            // per_rank_actual_token[rank]
  int64_t vecs_per_row;
  int vec_shift;                           // log2(vecs_per_row) or -1
  int ntensors;
  int n_dst;
  int64_t num_slots;
};

template <bool kPow2>
__global__ void __launch_bounds__(kThreads) push_rows_kernel(const __grid_constant__ PushArgs a) {
  const int64_t per_tensor = a.rows * a.vecs_per_row;
  const int64_t total = per_tensor * a.ntensors;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t vmask = a.vecs_per_row - 1;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride * kUnroll) {
    int4 val[kUnroll];
    int64_t tok[kUnroll], vec[kUnroll] = {};
    int which[kUnroll] = {};
    // Loads first (they depend only on the local row), stores after.
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = i + u * stride;
      tok[u] = -1;
      if (e < total) {
        which[u] = e >= per_tensor ? 1 : 0;
        const int64_t f = which[u] ? e - per_tensor : e;
        const int64_t row = kPow2 ? (f >> a.vec_shift) : f / a.vecs_per_row;
        vec[u] = kPow2 ? (f & vmask) : f - row * a.vecs_per_row;
        tok[u] = __ldg(a.tok + row);
        val[u] = ld_stream(a.src[which[u]] + (kPow2 ? (row << a.vec_shift) : row * a.vecs_per_row) + vec[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (tok[u] < 0) continue;
      for (int j = 0; j < a.n_dst; ++j) {
        const int64_t slot = __ldg(a.loc[j] + tok[u]);
        if (slot < 0 || slot >= a.num_slots) continue;
        int4* d = a.dst[which[u]][j] + (kPow2 ? (slot << a.vec_shift) : slot * a.vecs_per_row) + vec[u];
        *d = val[u];
      }
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int pow2_shift(int64_t x) {
  if (x <= 0 || (x & (x - 1))) return -1;
  int s = 0;
  while ((int64_t(1) << s) < x) ++s;
  return s;
}

PFN_cuMemGetAddressRange_v3020 g_get_range = nullptr;

zz_status_t get_range_fn() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* fn = nullptr;
    err = cudaGetDriverEntryPoint("cuMemGetAddressRange", &fn, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_get_range = reinterpret_cast<PFN_cuMemGetAddressRange_v3020>(fn);
  });
  if (!g_get_range)
    return zz::fail(ZZ_ERR_CUDA, std::string("cuMemGetAddressRange unavailable: ") + cudaGetErrorString(err));
  return ZZ_OK;
}

}  // namespace

extern "C" zz_status_t zz_rerange_push_kv(const zz_plan_t* plan, int rank, const void* k_local,
                                          const void* v_local, void* const* k_pools,
                                          void* const* v_pools, const int64_t* const* out_cache_locs,
                                          int n_dst, int64_t num_slots, int h_kv, int d,
                                          zz_dtype_t dtype, void* stream) {
  ZZ_NVTX("zz_rerange_push_kv");
  if (!plan || !k_local || !k_pools || !out_cache_locs)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: NULL argument");
  if ((v_local == nullptr) != (v_pools == nullptr))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: v_local and v_pools must both be set or both NULL");
  if (!plan->dev_ws) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: plan not uploaded");
  if (rank < 0 || rank >= plan->c) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: rank out of range");
  if (n_dst < 1 || n_dst > ZZ_MAX_PUSH_DST)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: n_dst must be in [1, ZZ_MAX_PUSH_DST]");
  if (h_kv <= 0 || d <= 0 || num_slots < 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: bad sizes");
  int64_t esize;
  switch (dtype) {
    case ZZ_BF16: esize = 2; break;
    case ZZ_FP32: esize = 4; break;
    default: return zz::fail(ZZ_ERR_UNSUPPORTED, "zz_rerange_push_kv: dtype");
  }
  const int64_t row_bytes = int64_t(h_kv) * d * esize;
  if (row_bytes % 16)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: h_kv*d*sizeof(dtype) must be a multiple of 16");
  PushArgs a{};
  a.ntensors = v_local ? 2 : 1;
  a.src[0] = static_cast<const int4*>(k_local);
  a.src[1] = static_cast<const int4*>(v_local);
  if (!aligned16(k_local) || (v_local && !aligned16(v_local)))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: pointers must be 16-byte aligned");
  for (int j = 0; j < n_dst; ++j) {
    if (!k_pools[j] || !out_cache_locs[j] || (v_pools && !v_pools[j]))
      return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: NULL destination pointer");
    if (!aligned16(k_pools[j]) || (v_pools && !aligned16(v_pools[j])))
      return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_push_kv: pointers must be 16-byte aligned");
    a.dst[0][j] = static_cast<int4*>(k_pools[j]);
    a.dst[1][j] = v_pools ? static_cast<int4*>(v_pools[j]) : nullptr;
    a.loc[j] = out_cache_locs[j];
  }
  a.n_dst = n_dst;
  a.tok = reinterpret_cast<const int32_t*>(static_cast<const char*>(plan->dev_ws) + plan->ws.rank_tok) +
          int64_t(rank) * plan->M;
  a.rows = plan->per_rank[rank];
  a.vecs_per_row = row_bytes / 16;
  a.vec_shift = pow2_shift(a.vecs_per_row);
  a.num_slots = num_slots;
  const int64_t total = a.rows * a.vecs_per_row * a.ntensors;
  if (total == 0) return ZZ_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = int64_t(sms) * 8;
  const int64_t need = (total + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
  if (need < blocks) blocks = need;
  auto s = static_cast<cudaStream_t>(stream);
  if (a.vec_shift >= 0) push_rows_kernel<true><<<unsigned(blocks), kThreads, 0, s>>>(a);
  else push_rows_kernel<false><<<unsigned(blocks), kThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("push_rows launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}

extern "C" zz_status_t zz_ipc_export(const void* dev_ptr, void* handle, int64_t* offset) {
  if (!dev_ptr || !handle || !offset) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_ipc_export: NULL argument");
  if (zz_status_t st = get_range_fn()) return st;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (g_get_range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return zz::fail(ZZ_ERR_CUDA, "zz_ipc_export: pointer is not inside a device allocation");
  cudaIpcMemHandle_t h;
  cudaError_t e = cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("zz_ipc_export: ") + cudaGetErrorString(e));
  static_assert(sizeof(h) == ZZ_IPC_HANDLE_BYTES, "IPC handle size");
  std::memcpy(handle, &h, sizeof(h));
  *offset = int64_t(reinterpret_cast<uintptr_t>(dev_ptr) - uintptr_t(base));
  return ZZ_OK;
}

extern "C" zz_status_t zz_ipc_import(const void* handle, int64_t offset, void** base, void** dev_ptr) {
  if (!handle || !base || !dev_ptr) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_ipc_import: NULL argument");
  if (offset < 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_ipc_import: negative offset");
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  void* b = nullptr;
  cudaError_t e = cudaIpcOpenMemHandle(&b, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("zz_ipc_import: ") + cudaGetErrorString(e));
  *base = b;
  *dev_ptr = static_cast<char*>(b) + offset;
  return ZZ_OK;
}

extern "C" zz_status_t zz_ipc_close(void* base) {
  if (!base) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_ipc_close: NULL argument");
  cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("zz_ipc_close: ") + cudaGetErrorString(e));
  return ZZ_OK;
}
