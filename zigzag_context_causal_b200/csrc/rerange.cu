// Row movement kernels: the fused K/V rerange into the paged pool, and the
// natural -> rank-ordered shard.  Pure data movement, bound by HBM bandwidth.
//
// rerange (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// _all_gather_reorganized + gather_kv_cache + materialize_full_kv): the page
// pads, all-gathers, trims, splits, concatenates and then scatters into the
// pool — four passes over K/V.  Here the trim, the reverse split/cat and the
// pool write collapse into one gather-scatter per 16-byte vector:
//     pool[out_cache_loc[t]] = gathered[src_row[t]],
// with src_row (natural token -> padded rank-ordered row) precomputed by the
// host planner.  Every byte is read once and written once.
#include <cuda_runtime.h>

#include <string>

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

__device__ __forceinline__ void st_stream(int4* p, int4 v) {
  asm volatile("st.global.cs.v4.s32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// One launch moves `ntensors` (1 or 2) tensors of `rows` rows each.  Vector v
// of the flattened [tensor][row][vec] space: dst row = dst_map(row), src row =
// src_map(row).  `vec_shift` = log2(vectors per row) when that is a power of
// two, else -1.
struct MoveArgs {
  const int4* src[2];
  int4* dst[2];
  const int32_t* src_idx;  // nullptr = identity
  const int32_t* dst_idx32;  // one of dst_idx32 / dst_idx64 / neither (identity)
  const int64_t* dst_idx64;
  int64_t rows;
  int64_t vecs_per_row;
  int vec_shift;
  int ntensors;
  int64_t dst_rows;  // rows of the destination, out-of-range rows are skipped
};

__global__ void __launch_bounds__(kThreads) move_rows_kernel(MoveArgs a) {
  const int64_t per_tensor = a.rows * a.vecs_per_row;
  const int64_t total = per_tensor * a.ntensors;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i < total; i += stride * kUnroll) {
    int4 val[kUnroll];
    int4* dptr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = i + u * stride;
      dptr[u] = nullptr;
      if (e < total) {
        const int tsel = e >= per_tensor;
        const int64_t f = e - (tsel ? per_tensor : 0);
        int64_t row, vec;
        if (a.vec_shift >= 0) {
          row = f >> a.vec_shift;
          vec = f & (a.vecs_per_row - 1);
        } else {
          row = f / a.vecs_per_row;
          vec = f - row * a.vecs_per_row;
        }
        const int64_t srow = a.src_idx ? int64_t(__ldg(a.src_idx + row)) : row;
        const int64_t drow = a.dst_idx64 ? __ldg(a.dst_idx64 + row)
                             : a.dst_idx32 ? int64_t(__ldg(a.dst_idx32 + row)) : row;
        if (drow >= 0 && drow < a.dst_rows) {
          const int4* sb = tsel ? a.src[1] : a.src[0];
          int4* db = tsel ? a.dst[1] : a.dst[0];
          val[u] = ld_stream(sb + srow * a.vecs_per_row + vec);
          dptr[u] = db + drow * a.vecs_per_row + vec;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dptr[u]) st_stream(dptr[u], val[u]);
  }
}

zz_status_t launch_move(const MoveArgs& a, cudaStream_t s) {
  const int64_t total = a.rows * a.vecs_per_row * a.ntensors;
  if (total == 0) return ZZ_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // 8 resident blocks of 256 threads per SM, 4 vectors in flight per thread.
  int64_t blocks = int64_t(sms) * 8;
  const int64_t need = (total + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
  if (need < blocks) blocks = need;
  move_rows_kernel<<<unsigned(blocks), kThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("move_rows launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int pow2_shift(int64_t x) {
  if (x <= 0 || (x & (x - 1))) return -1;
  int s = 0;
  while ((int64_t(1) << s) < x) ++s;
  return s;
}

}  // namespace

extern "C" zz_status_t zz_shard_rows(const zz_plan_t* plan, const void* src, void* dst,
                                     int64_t row_bytes, void* stream) {
  if (!plan || !src || !dst) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_shard_rows: NULL argument");
  if (!plan->dev_ws) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_shard_rows: plan not uploaded");
  if (row_bytes <= 0 || row_bytes % 16)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_shard_rows: row_bytes must be a positive multiple of 16");
  if (!aligned16(src) || !aligned16(dst))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_shard_rows: pointers must be 16-byte aligned");
  MoveArgs a{};
  a.src[0] = static_cast<const int4*>(src);
  a.dst[0] = static_cast<int4*>(dst);
  a.src_idx = nullptr;
  a.dst_idx32 = reinterpret_cast<const int32_t*>(static_cast<const char*>(plan->dev_ws) + plan->ws.src_row);
  a.rows = plan->T;
  a.vecs_per_row = row_bytes / 16;
  a.vec_shift = pow2_shift(a.vecs_per_row);
  a.ntensors = 1;
  a.dst_rows = int64_t(plan->c) * plan->M;
  return launch_move(a, static_cast<cudaStream_t>(stream));
}

extern "C" zz_status_t zz_rerange_kv_to_pool(const zz_plan_t* plan, const void* k_gathered,
                                             const void* v_gathered, void* k_pool, void* v_pool,
                                             const int64_t* out_cache_loc, int64_t num_slots,
                                             int h_kv, int d, zz_dtype_t dtype, void* stream) {
  if (!plan || !k_gathered || !k_pool || !out_cache_loc)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: NULL argument");
  if ((v_gathered == nullptr) != (v_pool == nullptr))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: v_gathered and v_pool must both be set or both NULL");
  if (!plan->dev_ws) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: plan not uploaded");
  if (h_kv <= 0 || d <= 0 || num_slots < 0)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: bad sizes");
  int64_t esize;
  switch (dtype) {
    case ZZ_BF16: esize = 2; break;
    case ZZ_FP32: esize = 4; break;
    default: return zz::fail(ZZ_ERR_UNSUPPORTED, "zz_rerange_kv_to_pool: dtype");
  }
  const int64_t row_bytes = int64_t(h_kv) * d * esize;
  if (row_bytes % 16)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: h_kv*d*sizeof(dtype) must be a multiple of 16");
  if (!aligned16(k_gathered) || !aligned16(k_pool) || (v_gathered && (!aligned16(v_gathered) || !aligned16(v_pool))))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool: pointers must be 16-byte aligned");
  MoveArgs a{};
  a.src[0] = static_cast<const int4*>(k_gathered);
  a.dst[0] = static_cast<int4*>(k_pool);
  a.src[1] = static_cast<const int4*>(v_gathered);
  a.dst[1] = static_cast<int4*>(v_pool);
  a.ntensors = v_gathered ? 2 : 1;
  a.src_idx = reinterpret_cast<const int32_t*>(static_cast<const char*>(plan->dev_ws) + plan->ws.src_row);
  a.dst_idx64 = out_cache_loc;
  a.rows = plan->T;
  a.vecs_per_row = row_bytes / 16;
  a.vec_shift = pow2_shift(a.vecs_per_row);
  a.dst_rows = num_slots;
  return launch_move(a, static_cast<cudaStream_t>(stream));
}
