// The fused K/V rerange into the paged pool.  Pure data movement, bound by
// HBM bandwidth.  (Token-order shard / gather / take-back live in permute.cu.)
//
// rerange (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// _all_gather_reorganized + gather_kv_cache + materialize_full_kv): the page
// pads, all-gathers, trims, splits, concatenates and then scatters into the
// pool — four passes over K/V.  Here the trim, the reverse split/cat and the
// pool write collapse into one gather-scatter of rows:
//     pool[out_cache_loc[t]] = gathered[src_row[t]],
// with src_row (natural token -> padded rank-ordered row) precomputed by the
// host planner.  Every byte is read once and written once: rows of 1-16 KB
// move whole through shared memory by the copy engine (move_rows_bulk), other
// rows as 16-byte vectors (move_rows_kernel).
#include <cuda_runtime.h>

#include <algorithm>
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

__device__ __forceinline__ void st_stream(int4* p, int4 v) {
  asm volatile("st.global.cs.v4.s32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// One launch moves `ntensors` (1 or 2) tensors of `rows` rows each.  Vector e
// of the flattened [tensor][row][vec] space goes from row src_map(row) of the
// source to row dst_map(row) of the destination.  The maps are compile-time
// choices (identity, int32 table, int64 table) so that the per-vector work is
// a shift, a mask, two cached index loads and the 16-byte copy.
struct MoveArgs {
  const int4* src[2];
  int4* dst[2];
  const int32_t* src_idx;    // natural token -> source row (nullptr: identity)
  const int32_t* dst_idx32;  // destination row tables (one of them, or identity)
  const int64_t* dst_idx64;
  int64_t rows;
  int64_t vecs_per_row;
  int vec_shift;             // log2(vecs_per_row), or -1 when not a power of two
  int ntensors;
  int64_t dst_rows;          // rows of the destination; out-of-range rows are skipped
  int* status;               // plan status word (bulk form: kStatusTimeout if a wait gave up)
};

enum DstKind { kDstIdentity = 0, kDstI32 = 1, kDstI64 = 2 };

template <bool kSrcTable, int kDst, bool kPow2>
__global__ void __launch_bounds__(kThreads) move_rows_kernel(MoveArgs a) {
  const int64_t per_tensor = a.rows * a.vecs_per_row;
  const int64_t total = per_tensor * a.ntensors;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t vmask = a.vecs_per_row - 1;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride * kUnroll) {
    int4 val[kUnroll];
    int4* dptr[kUnroll];
    // The 16-byte load depends only on the source index (rows of the plan,
    // valid by construction); the destination index is checked only to
    // predicate the store, so loads never wait on it.
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = i + u * stride;
      dptr[u] = nullptr;
      if (e < total) {
        const bool second = e >= per_tensor;
        const int64_t f = second ? e - per_tensor : e;
        const int64_t row = kPow2 ? (f >> a.vec_shift) : f / a.vecs_per_row;
        const int64_t vec = kPow2 ? (f & vmask) : f - row * a.vecs_per_row;
        const int64_t srow = kSrcTable ? int64_t(__ldg(a.src_idx + row)) : row;
        const int64_t drow = kDst == kDstI64 ? __ldg(a.dst_idx64 + row)
                             : kDst == kDstI32 ? int64_t(__ldg(a.dst_idx32 + row)) : row;
        const int4* sb = second ? a.src[1] : a.src[0];
        int4* db = second ? a.dst[1] : a.dst[0];
        const int64_t soff = kPow2 ? (srow << a.vec_shift) : srow * a.vecs_per_row;
        const int64_t doff = kPow2 ? (drow << a.vec_shift) : drow * a.vecs_per_row;
        val[u] = ld_stream(sb + soff + vec);
        if (kDst == kDstIdentity || (drow >= 0 && drow < a.dst_rows)) dptr[u] = db + doff + vec;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      if (dptr[u]) st_stream(dptr[u], val[u]);
  }
}

// ---- whole rows through shared memory, by the copy engine (cp.async.bulk) ----
// For rows of kBulkMinRow..kBulkMaxRow bytes.  A CTA is one warp that owns a
// contiguous range of the flattened [tensor][token] rows and keeps kBulkStages
// stages of about kBulkStageBytes each in flight: rows are loaded global ->
// shared (completion counted on the stage's mbarrier) and stored shared ->
// global as soon as they land; a stage is reloaded once the stores of the
// stage before have read it.  One warp per CTA and as many CTAs per SM as fit
// keep many independent copies in flight.  Measured against the 16-byte
// vector copy on K and V [32768, h_kv, 128] bf16 -> page-16 pool: 47.7 vs
// 48.7 us at 2 KB rows, 24.0 vs 25.5 us at 1 KB rows, 169 vs 191 us at 8 KB
// rows; 256-byte rows stay on the vector copy (8.3 vs 7.2 us).
constexpr uint32_t kBulkMinRow = 1024;
constexpr uint32_t kBulkMaxRow = 16 * 1024;        // two stages of one row fit the default 48 KB
constexpr uint32_t kBulkStageBytes = 8192;
constexpr int kBulkStages = 2;
constexpr int kBulkMaxRowsPerStage = int(kBulkStageBytes / kBulkMinRow);
constexpr uint64_t kBulkTimeoutNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for phase `parity` of an mbarrier.
__device__ __forceinline__ bool bulk_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = now_ns();
  for (uint32_t it = 0;; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_u32addr(bar)), "r"(parity)
        : "memory");
    if (done) return true;
    if ((it & 255u) == 255u && now_ns() - t0 > kBulkTimeoutNs) return false;
  }
}

__global__ void __launch_bounds__(32) move_rows_bulk(MoveArgs a, int R, uint32_t row_bytes) {
  extern __shared__ __align__(128) uint8_t stage_mem[];
  __shared__ __align__(8) uint64_t full[kBulkStages];
  __shared__ int64_t slot_dst[kBulkStages * kBulkMaxRowsPerStage];   // -1: row not stored
  const int lane = threadIdx.x;
  const int64_t total = a.rows * a.ntensors;
  const int64_t per_cta = (total + gridDim.x - 1) / gridDim.x;
  const int64_t start = int64_t(blockIdx.x) * per_cta;
  const int64_t end = min(start + per_cta, total);
  if (start >= end) return;
  const int64_t nb = (end - start + R - 1) / R;      // stages' worth of rows of this CTA
  if (lane == 0) {
    for (int s = 0; s < kBulkStages; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32addr(&full[s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  // Row i of batch b is handled by lane i % 32 for both its load and its
  // store, so each lane's own bulk groups cover the shared memory it reloads.
  auto load_batch = [&](int64_t b) {
    const int s = int(b % kBulkStages);
    const int64_t w0 = start + b * R;
    const int n = int(min(int64_t(R), end - w0));
    if (lane == 0)
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;"
                   ::"r"(smem_u32addr(&full[s])), "r"(uint32_t(n) * row_bytes) : "memory");
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const int64_t w = w0 + i;
      const bool second = w >= a.rows;
      const int64_t row = second ? w - a.rows : w;
      const int64_t srow = __ldg(a.src_idx + row);
      const int64_t drow = __ldg(a.dst_idx64 + row);
      slot_dst[s * kBulkMaxRowsPerStage + i] = (drow >= 0 && drow < a.dst_rows) ? drow : -1;
      const char* src = reinterpret_cast<const char*>(second ? a.src[1] : a.src[0]) + srow * int64_t(row_bytes);
      uint8_t* dst = stage_mem + (size_t(s) * R + i) * row_bytes;
      asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                   ::"r"(smem_u32addr(dst)), "l"(src), "r"(row_bytes), "r"(smem_u32addr(&full[s]))
                   : "memory");
    }
  };
  auto store_batch = [&](int64_t b) {
    const int s = int(b % kBulkStages);
    const int64_t w0 = start + b * R;
    const int n = int(min(int64_t(R), end - w0));
    for (int i = lane; i < n; i += 32) {
      const int64_t drow = slot_dst[s * kBulkMaxRowsPerStage + i];
      if (drow < 0) continue;
      const bool second = w0 + i >= a.rows;
      char* dst = reinterpret_cast<char*>(second ? a.dst[1] : a.dst[0]) + drow * int64_t(row_bytes);
      const uint8_t* src = stage_mem + (size_t(s) * R + i) * row_bytes;
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                   ::"l"(dst), "r"(smem_u32addr(src)), "r"(row_bytes) : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  };
  for (int64_t b = 0; b < nb && b < kBulkStages; ++b) load_batch(b);
  int64_t b = 0;
  bool ok = true;
  for (; b < nb; ++b) {
    ok = __all_sync(0xffffffffu, bulk_wait(&full[b % kBulkStages], uint32_t(b / kBulkStages) & 1u));
    if (!ok) break;
    store_batch(b);
    if (b >= 1 && b - 1 + kBulkStages < nb) {
      // the stores of batch b-1 have read its stage (the lane's groups but the newest)
      asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
      __syncwarp();
      load_batch(b - 1 + kBulkStages);
    }
  }
  if (!ok) {
    // Let the loads still in flight land before the CTA's shared memory goes.
    const int64_t issued = min(nb, b == 0 ? int64_t(kBulkStages) : b - 1 + kBulkStages);
    for (int64_t k = b; k < issued; ++k)
      bulk_wait(&full[k % kBulkStages], uint32_t(k / kBulkStages) & 1u);
    if (lane == 0 && a.status) atomicOr(a.status, zz::kStatusTimeout);
  }
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

template <bool kSrcTable, int kDst>
void launch_kind(const MoveArgs& a, unsigned blocks, cudaStream_t s) {
  if (a.vec_shift >= 0) move_rows_kernel<kSrcTable, kDst, true><<<blocks, kThreads, 0, s>>>(a);
  else move_rows_kernel<kSrcTable, kDst, false><<<blocks, kThreads, 0, s>>>(a);
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
  const unsigned b = unsigned(blocks);
  const int64_t row_bytes = a.vecs_per_row * 16;
  if (!(a.src_idx && a.dst_idx64)) return zz::fail(ZZ_ERR_INVALID_ARG, "move_rows: unsupported index maps");
  if (row_bytes >= kBulkMinRow && row_bytes <= kBulkMaxRow) {
    // Rerange into the pool, whole rows by the copy engine: stages of ~8 KB,
    // as many one-warp CTAs per SM as 220 KB of shared memory holds (<= 16).
    const int R = int(std::max<int64_t>(1, kBulkStageBytes / row_bytes));
    const size_t smem = size_t(kBulkStages) * R * size_t(row_bytes);
    const int per_sm = int(std::min<size_t>(16, (220u * 1024u) / (smem + 1024u)));
    const int64_t rows = a.rows * a.ntensors;
    const int64_t grid = std::min<int64_t>(int64_t(sms) * per_sm, (rows + R - 1) / R);
    move_rows_bulk<<<unsigned(grid), 32, smem, s>>>(a, R, uint32_t(row_bytes));
  } else {
    launch_kind<true, kDstI64>(a, b, s);                                         // rerange into the pool
  }
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

extern "C" zz_status_t zz_rerange_kv_to_pool(const zz_plan_t* plan, const void* k_gathered,
                                             const void* v_gathered, void* k_pool, void* v_pool,
                                             const int64_t* out_cache_loc, int64_t num_slots,
                                             int h_kv, int d, zz_dtype_t dtype, void* stream) {
  ZZ_NVTX("zz_rerange_kv_to_pool");
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
  a.status = reinterpret_cast<int*>(static_cast<char*>(plan->dev_ws) + plan->ws.status);
  return launch_move(a, static_cast<cudaStream_t>(stream));
}
