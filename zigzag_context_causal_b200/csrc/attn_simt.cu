// CUDA-core zigzag prefill attention in full fp32 (the fp32 dtype of
// zz_attn_prefill).  One CTA = one 128-row query tile of one half and one
// query head; one thread = one query row; keys stream through shared memory
// in chunks of 32 with an online (running max / running sum) softmax.
// Same work list, half table and paged K/V addressing as the tensor-core
// kernel; the page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// run_attention, defines the per-half problem.
#include <cuda_runtime.h>
#include <math_constants.h>

#include <string>

#include "zz_internal.h"

namespace zz {
namespace {

constexpr int kChunk = 32;

struct SimtArgs {
  const float* q;
  const float* k_pool;
  const float* v_pool;
  const int32_t* page_table;
  float* out;
  float* lse;
  const HalfDesc* halves;
  const WorkItem* items;
  int64_t num_slots;
  int max_pages, page_size;
  int h_q, h_kv, group;
  int M, rank_begin;
  float scale;
  int causal;
  int* status;          // device status word (kStatusBadPage)
};

template <int D>
__global__ void __launch_bounds__(kTileM) attn_simt_kernel(SimtArgs a) {
  __shared__ float ks[kChunk][D];
  __shared__ float vs[kChunk][D];
  const WorkItem w = a.items[blockIdx.x / a.h_q];
  const int head = blockIdx.x % a.h_q;
  const int kvh = head / a.group;
  const HalfDesc hd = a.halves[w.half_id];
  const int q0 = w.tile * kTileM;
  const int row = q0 + threadIdx.x;
  const bool valid = row < hd.lq;
  const int64_t grow = int64_t(hd.rank - a.rank_begin) * a.M + hd.row0 + row;
  float qv[D], o[D];
  if (valid) {
    const float* qp = a.q + (grow * a.h_q + head) * D;
#pragma unroll
    for (int i = 0; i < D; ++i) qv[i] = qp[i] * a.scale;
  } else {
#pragma unroll
    for (int i = 0; i < D; ++i) qv[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < D; ++i) o[i] = 0.f;
  float m = -CUDART_INF_F, l = 0.f;
  // Inclusive last key of my row and of the CTA; without the causal mask every
  // row sees the whole sequence (kv_full keys).
  const int kv_end = a.causal ? hd.kv_len : hd.kv_full;
  const int my_last = a.causal ? hd.kv_pos0 + row : hd.kv_full - 1;
  const int tile_last_row = min(q0 + kTileM, hd.lq) - 1;
  const int cta_last = a.causal ? hd.kv_pos0 + tile_last_row : hd.kv_full - 1;
  const int32_t* pt = a.page_table + int64_t(hd.seq) * a.max_pages;
  bool bad_page = false;   // a page outside the pool: its keys read as zeros, reported in status
  for (int k0 = 0; k0 <= cta_last; k0 += kChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kChunk * D; e += blockDim.x) {
      const int j = e / D, x = e % D;
      const int key = k0 + j;
      float kx = 0.f, vx = 0.f;
      if (key < kv_end) {
        const int64_t slot = int64_t(pt[key / a.page_size]) * a.page_size + key % a.page_size;
        if (slot >= 0 && slot < a.num_slots) {
          const int64_t off = (slot * a.h_kv + kvh) * D + x;
          kx = a.k_pool[off];
          vx = a.v_pool[off];
        } else {
          bad_page = true;
        }
      }
      ks[j][x] = kx;
      vs[j][x] = vx;
    }
    __syncthreads();
    float s[kChunk];
    float cmax = -CUDART_INF_F;
#pragma unroll 4
    for (int j = 0; j < kChunk; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < D; ++i) acc = fmaf(qv[i], ks[j][i], acc);
      s[j] = (k0 + j <= my_last) ? acc : -CUDART_INF_F;
      cmax = fmaxf(cmax, s[j]);
    }
    const float m_new = fmaxf(m, cmax);
    if (m_new == -CUDART_INF_F) continue;                    // nothing visible yet
    const float corr = expf(m - m_new);
    l *= corr;
#pragma unroll
    for (int i = 0; i < D; ++i) o[i] *= corr;
#pragma unroll 4
    for (int j = 0; j < kChunk; ++j) {
      const float p = expf(s[j] - m_new);
      l += p;
#pragma unroll
      for (int i = 0; i < D; ++i) o[i] = fmaf(p, vs[j][i], o[i]);
    }
    m = m_new;
  }
  if (bad_page && a.status) atomicOr(a.status, kStatusBadPage);
  if (!valid) return;
  const float inv = 1.f / l;
  float* op = a.out + (grow * a.h_q + head) * D;
#pragma unroll
  for (int i = 0; i < D; ++i) op[i] = o[i] * inv;
  if (a.lse) a.lse[grow * a.h_q + head] = m + logf(l);
}

}  // namespace

zz_status_t launch_attn_simt_fp32(const zz_plan_t* p, int rank_begin, int rank_count,
                                  const void* q, const void* k_pool, const void* v_pool,
                                  int64_t num_slots, const int32_t* page_table, int max_pages,
                                  int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                                  float scale, int causal, cudaStream_t s) {
  const char* ws = static_cast<const char*>(p->dev_ws);
  SimtArgs a{};
  a.q = static_cast<const float*>(q);
  a.k_pool = static_cast<const float*>(k_pool);
  a.v_pool = static_cast<const float*>(v_pool);
  a.page_table = page_table;
  a.out = static_cast<float*>(out);
  a.lse = lse;
  a.halves = reinterpret_cast<const HalfDesc*>(ws + p->ws.halves);
  int64_t n_items;
  if (rank_count == p->c) {
    a.items = reinterpret_cast<const WorkItem*>(ws + p->ws.tiles_all);
    n_items = int64_t(p->tiles_all.size());
  } else {
    a.items = reinterpret_cast<const WorkItem*>(ws + p->ws.tiles_rank) + p->tile_rank_off[rank_begin];
    n_items = p->tile_rank_off[rank_begin + rank_count] - p->tile_rank_off[rank_begin];
  }
  a.num_slots = num_slots;
  a.max_pages = max_pages;
  a.page_size = page_size;
  a.h_q = h_q;
  a.h_kv = h_kv;
  a.group = h_q / h_kv;
  a.M = p->M;
  a.rank_begin = rank_begin;
  a.scale = scale;
  a.causal = causal;
  a.status = reinterpret_cast<int*>(const_cast<char*>(ws) + p->ws.status);
  const int64_t grid = n_items * h_q;
  if (grid == 0) return ZZ_OK;
  if (grid > INT32_MAX) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: grid too large");
  if (d == 64) attn_simt_kernel<64><<<unsigned(grid), kTileM, 0, s>>>(a);
  else attn_simt_kernel<128><<<unsigned(grid), kTileM, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("attn_simt launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}

}  // namespace zz
