// Fused K/V rerange into an FP8 (E4M3) paged pool with per-tensor scales
// (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// materialize_full_kv: set_kv_buffer receives layer.k_scale / layer.v_scale).
//     pool_K[out_cache_loc[t]] = e4m3(gathered_K[src_row[t]] / k_scale)
// and the same for V; the division is rounded in fp32, the conversion rounds
// to nearest even and saturates finite overflow at +-448.  bf16 in, 1 byte
// out: each thread turns 32 bytes of input into one 16-byte store.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <string>

#include "nvtx_range.h"
#include "zz_internal.h"

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 2;

struct Fp8Args {
  const int4* src[2];    // bf16 rows, 16 elements = 2 x int4
  int4* dst[2];          // e4m3 rows, 16 elements = 1 x int4
  const int32_t* src_row;
  const int64_t* loc;
  float scale[2];
  int64_t rows;
  int64_t groups;        // 16-element groups per row
  int ntensors;
  int64_t num_slots;
};

__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 8 bf16 values (one int4) -> 8 e4m3 bytes (two uint32)
__device__ __forceinline__ uint2 convert8(int4 v, float s) {
  const uint32_t w[4] = {uint32_t(v.x), uint32_t(v.y), uint32_t(v.z), uint32_t(v.w)};
  uint32_t b[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float lo = __uint_as_float(w[i] << 16);
    const float hi = __uint_as_float(w[i] & 0xFFFF0000u);
    b[i] = e4m3x2(__fdiv_rn(lo, s), __fdiv_rn(hi, s));
  }
  return make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
}

__global__ void __launch_bounds__(kThreads) rerange_fp8_kernel(Fp8Args a) {
  const int64_t per_tensor = a.rows * a.groups;
  const int64_t total = per_tensor * a.ntensors;
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride * kUnroll) {
    int4 in[kUnroll][2];
    int4* dptr[kUnroll];
    float sc[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t e = i + u * stride;
      dptr[u] = nullptr;
      if (e < total) {
        const bool second = e >= per_tensor;
        const int64_t f = second ? e - per_tensor : e;
        const int64_t t = f / a.groups;
        const int64_t grp = f - t * a.groups;
        const int64_t srow = __ldg(a.src_row + t);
        const int64_t slot = __ldg(a.loc + t);
        const int4* s = (second ? a.src[1] : a.src[0]) + (srow * a.groups + grp) * 2;
        in[u][0] = __ldg(s);
        in[u][1] = __ldg(s + 1);
        sc[u] = second ? a.scale[1] : a.scale[0];
        if (slot >= 0 && slot < a.num_slots) dptr[u] = (second ? a.dst[1] : a.dst[0]) + slot * a.groups + grp;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (!dptr[u]) continue;
      const uint2 lo = convert8(in[u][0], sc[u]);
      const uint2 hi = convert8(in[u][1], sc[u]);
      *dptr[u] = make_int4(int(lo.x), int(lo.y), int(hi.x), int(hi.y));
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" zz_status_t zz_rerange_kv_to_pool_fp8(const zz_plan_t* plan, const void* k_gathered,
                                                 const void* v_gathered, void* k_pool, void* v_pool,
                                                 const int64_t* out_cache_loc, int64_t num_slots,
                                                 int h_kv, int d, float k_scale, float v_scale,
                                                 void* stream) {
  ZZ_NVTX("zz_rerange_kv_to_pool_fp8");
  if (!plan || !k_gathered || !k_pool || !out_cache_loc)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: NULL argument");
  if ((v_gathered == nullptr) != (v_pool == nullptr))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: v_gathered and v_pool must both be set or both NULL");
  if (!plan->dev_ws) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: plan not uploaded");
  if (h_kv <= 0 || d <= 0 || num_slots < 0 || (int64_t(h_kv) * d) % 16)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: h_kv*d must be a positive multiple of 16");
  if (!(k_scale > 0.f) || !std::isfinite(k_scale) || (v_gathered && (!(v_scale > 0.f) || !std::isfinite(v_scale))))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: scales must be positive and finite");
  if (!aligned16(k_gathered) || !aligned16(k_pool) || (v_gathered && (!aligned16(v_gathered) || !aligned16(v_pool))))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_rerange_kv_to_pool_fp8: pointers must be 16-byte aligned");
  Fp8Args a{};
  a.src[0] = static_cast<const int4*>(k_gathered);
  a.src[1] = static_cast<const int4*>(v_gathered);
  a.dst[0] = static_cast<int4*>(k_pool);
  a.dst[1] = static_cast<int4*>(v_pool);
  a.src_row = reinterpret_cast<const int32_t*>(static_cast<const char*>(plan->dev_ws) + plan->ws.src_row);
  a.loc = out_cache_loc;
  a.scale[0] = k_scale;
  a.scale[1] = v_scale;
  a.rows = plan->T;
  a.groups = int64_t(h_kv) * d / 16;
  a.ntensors = v_gathered ? 2 : 1;
  a.num_slots = num_slots;
  const int64_t total = a.rows * a.groups * a.ntensors;
  if (total == 0) return ZZ_OK;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = int64_t(sms) * 8;
  const int64_t need = (total + int64_t(kThreads) * kUnroll - 1) / (int64_t(kThreads) * kUnroll);
  if (need < blocks) blocks = need;
  rerange_fp8_kernel<<<unsigned(blocks), kThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return zz::fail(ZZ_ERR_CUDA, std::string("rerange_fp8 launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}
