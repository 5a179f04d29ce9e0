// Row permutations between token order and the rank-ordered zigzag layout
// (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py":
// shard_hidden_states / shard_position_ids, gather_hidden_states; and the
// take-back of one rank's shard from a token-order tensor).  Each is one pass
// over the rows with the plan's token -> row map; rows may be as small as 4
// bytes (position ids).
#include <cuda_runtime.h>

#include <string>

#include "nvtx_range.h"
#include "zz_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

// out row map: dst_row = table ? table[t] - offset : t;  in row map: src_row =
// table ? table[t] - offset : t.  Rows whose destination falls outside
// [0, dst_rows) are skipped (take-back keeps only this rank's rows).
struct PermuteArgs {
  const void* src;
  void* dst;
  const int32_t* table;   // plan: natural token -> rank-ordered row
  int64_t offset;         // subtracted from table values
  int table_on_dst;       // 1: scatter (dst = table), 0: gather (src = table)
  int64_t rows;           // tokens
  int64_t vecs_per_row;   // in units of V
  int64_t dst_rows;
};

template <typename V>
__global__ void __launch_bounds__(kThreads) permute_kernel(PermuteArgs a) {
  const int64_t total = a.rows * a.vecs_per_row;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const V* src = static_cast<const V*>(a.src);
  V* dst = static_cast<V*>(a.dst);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride * kUnroll) {
    V val[kUnroll];
    V* dptr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = i + u * stride;
      dptr[u] = nullptr;
      if (e < total) {
        const int64_t t = e / a.vecs_per_row;
        const int64_t vec = e - t * a.vecs_per_row;
        const int64_t mapped = int64_t(__ldg(a.table + t)) - a.offset;
        const int64_t srow = a.table_on_dst ? t : mapped;
        const int64_t drow = a.table_on_dst ? mapped : t;
        if (drow >= 0 && drow < a.dst_rows) {
          val[u] = __ldg(src + srow * a.vecs_per_row + vec);
          dptr[u] = dst + drow * a.vecs_per_row + vec;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dptr[u]) *dptr[u] = val[u];
  }
}

zz_status_t launch_permute(const char* who, const zz_plan_t* plan, const void* src, void* dst,
                           int64_t row_bytes, int64_t offset, int table_on_dst, int64_t dst_rows,
                           cudaStream_t s) {
  if (!plan || !src || !dst) return zz::fail(ZZ_ERR_INVALID_ARG, std::string(who) + ": NULL argument");
  if (!plan->dev_ws) return zz::fail(ZZ_ERR_INVALID_ARG, std::string(who) + ": plan not uploaded");
  if (row_bytes <= 0 || row_bytes % 4)
    return zz::fail(ZZ_ERR_INVALID_ARG, std::string(who) + ": row_bytes must be a positive multiple of 4");
  const bool wide = row_bytes % 16 == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                    (reinterpret_cast<uintptr_t>(dst) & 15) == 0;
  if ((reinterpret_cast<uintptr_t>(src) & 3) || (reinterpret_cast<uintptr_t>(dst) & 3))
    return zz::fail(ZZ_ERR_INVALID_ARG, std::string(who) + ": pointers must be 4-byte aligned");
  PermuteArgs a{};
  a.src = src;
  a.dst = dst;
  a.table = reinterpret_cast<const int32_t*>(static_cast<const char*>(plan->dev_ws) + plan->ws.src_row);
  a.offset = offset;
  a.table_on_dst = table_on_dst;
  a.rows = plan->T;
  a.vecs_per_row = row_bytes / (wide ? 16 : 4);
  a.dst_rows = dst_rows;
  const int64_t total = a.rows * a.vecs_per_row;
  if (total == 0) return ZZ_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = int64_t(sms) * 8;
  const int64_t need = (total + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
  if (need < blocks) blocks = need;
  if (wide) permute_kernel<int4><<<unsigned(blocks), kThreads, 0, s>>>(a);
  else permute_kernel<int><<<unsigned(blocks), kThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string(who) + ": " + cudaGetErrorString(e));
  return ZZ_OK;
}

}  // namespace

extern "C" zz_status_t zz_shard_rows(const zz_plan_t* plan, const void* src, void* dst,
                                     int64_t row_bytes, void* stream) {
  ZZ_NVTX("zz_shard_rows");
  if (!plan) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_shard_rows: NULL plan");
  return launch_permute("zz_shard_rows", plan, src, dst, row_bytes, 0, 1, int64_t(plan->c) * plan->M,
                        static_cast<cudaStream_t>(stream));
}

extern "C" zz_status_t zz_gather_rows(const zz_plan_t* plan, const void* src, void* dst,
                                      int64_t row_bytes, void* stream) {
  ZZ_NVTX("zz_gather_rows");
  if (!plan) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_gather_rows: NULL plan");
  return launch_permute("zz_gather_rows", plan, src, dst, row_bytes, 0, 0, plan->T,
                        static_cast<cudaStream_t>(stream));
}

extern "C" zz_status_t zz_take_back_rows(const zz_plan_t* plan, int rank, const void* src, void* dst,
                                         int64_t row_bytes, void* stream) {
  ZZ_NVTX("zz_take_back_rows");
  if (!plan) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_take_back_rows: NULL plan");
  if (rank < 0 || rank >= plan->c) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_take_back_rows: rank out of range");
  return launch_permute("zz_take_back_rows", plan, src, dst, row_bytes, int64_t(rank) * plan->M, 1,
                        plan->per_rank[rank], static_cast<cudaStream_t>(stream));
}
