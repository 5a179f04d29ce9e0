// CUDA-core zigzag prefill attention in full fp32 (the fp32 dtype of
// zz_attn_prefill).  One CTA = 32 rows of a 128-row query tile of one half and
// one query head (small CTAs spread the short fp32 problems over many SMs);
// four threads per query row, each owning D/4 of the head dimensions (partial
// dot products combined with two shuffles); keys stream through shared memory
// in chunks of 32, the next chunk loaded into registers while the current one
// is computed, with an online (running max / running sum) softmax.  Same work list, half table and paged K/V addressing as the
// tensor-core kernel; the page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// run_attention, defines the per-half problem.
#include <cuda_runtime.h>
#include <math_constants.h>

#include <string>

#include "zz_internal.h"

namespace zz {
namespace {

constexpr int kChunk = 32;
constexpr int kLanesPerRow = 4;
constexpr int kSimtRows = 32;                          // query rows per CTA
constexpr int kSimtThreads = kSimtRows * kLanesPerRow;
constexpr int kRowGroups = kTileM / kSimtRows;         // CTAs per tile and head

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
__global__ void __launch_bounds__(kSimtThreads) attn_simt_kernel(SimtArgs a) {
  constexpr int kDpt = D / kLanesPerRow;              // dims per thread
  __shared__ __align__(16) float ks[kChunk][D];
  __shared__ __align__(16) float vs[kChunk][D];
  const int rg = blockIdx.x % kRowGroups;
  const int head = (blockIdx.x / kRowGroups) % a.h_q;
  const WorkItem w = a.items[blockIdx.x / (kRowGroups * a.h_q)];
  const int kvh = head / a.group;
  const HalfDesc hd = a.halves[w.half_id];
  const int q0 = w.tile * kTileM + rg * kSimtRows;   // first row of this CTA
  if (q0 >= hd.lq) return;                           // the whole CTA is past the half
  const int sub = threadIdx.x & (kLanesPerRow - 1);   // which D/4 slice of the row
  const int row = q0 + (threadIdx.x >> 2);
  const int d0 = sub * kDpt;
  const bool valid = row < hd.lq;
  const int64_t grow = int64_t(hd.rank - a.rank_begin) * a.M + hd.row0 + row;
  // log2-domain scores: s * scale * log2(e), so that exp2f gives e^(s * scale)
  const float qscale = a.scale * 1.4426950408889634f;
  float qv[kDpt], o[kDpt];
  if (valid) {
    const float4* qp = reinterpret_cast<const float4*>(a.q + (grow * a.h_q + head) * D + d0);
#pragma unroll
    for (int i = 0; i < kDpt / 4; ++i) {
      const float4 x = qp[i];
      qv[4 * i] = x.x * qscale; qv[4 * i + 1] = x.y * qscale; qv[4 * i + 2] = x.z * qscale; qv[4 * i + 3] = x.w * qscale;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kDpt; ++i) qv[i] = 0.f;
  }
#pragma unroll
  for (int i = 0; i < kDpt; ++i) o[i] = 0.f;
  float m = -CUDART_INF_F, l = 0.f;
  // Inclusive last key of my row and of the CTA; without the causal mask every
  // row sees the whole sequence (kv_full keys).
  const int kv_end = a.causal ? hd.kv_len : hd.kv_full;
  const int my_last = a.causal ? hd.kv_pos0 + row : hd.kv_full - 1;
  const int tile_last_row = min(q0 + kSimtRows, hd.lq) - 1;
  const int cta_last = a.causal ? hd.kv_pos0 + tile_last_row : hd.kv_full - 1;
  const int32_t* pt = a.page_table + int64_t(hd.seq) * a.max_pages;
  bool bad_page = false;   // a page outside the pool: its keys read as zeros, reported in status
  // Each thread moves kPieces 16-byte pieces of K and of V per chunk.  The next
  // chunk's pieces are loaded into registers while the current chunk is
  // computed, so only the first chunk waits on memory (the page-table read and
  // the K/V read it feeds are dependent loads).
  constexpr int kPieces = kChunk * D / 4 / kSimtThreads;
  static_assert(kPieces * kSimtThreads == kChunk * D / 4, "pieces per thread");
  float4 kr[kPieces], vr[kPieces];
  auto fetch = [&](int k0) {
#pragma unroll
    for (int it = 0; it < kPieces; ++it) {
      const int e = threadIdx.x + it * kSimtThreads;
      const int key = k0 + e / (D / 4), x = (e % (D / 4)) * 4;
      kr[it] = make_float4(0.f, 0.f, 0.f, 0.f);
      vr[it] = kr[it];
      if (key < kv_end) {
        const int64_t slot = int64_t(pt[key / a.page_size]) * a.page_size + key % a.page_size;
        if (slot >= 0 && slot < a.num_slots) {
          const int64_t off = (slot * a.h_kv + kvh) * D + x;
          kr[it] = *reinterpret_cast<const float4*>(a.k_pool + off);
          vr[it] = *reinterpret_cast<const float4*>(a.v_pool + off);
        } else {
          bad_page = true;
        }
      }
    }
  };
  fetch(0);
  for (int k0 = 0; k0 <= cta_last; k0 += kChunk) {
    __syncthreads();                       // the previous chunk is no longer read
#pragma unroll
    for (int it = 0; it < kPieces; ++it) {
      const int e = threadIdx.x + it * kSimtThreads;
      const int j = e / (D / 4), x = (e % (D / 4)) * 4;
      *reinterpret_cast<float4*>(&ks[j][x]) = kr[it];
      *reinterpret_cast<float4*>(&vs[j][x]) = vr[it];
    }
    __syncthreads();
    if (k0 + kChunk <= cta_last) fetch(k0 + kChunk);
    float s[kChunk];
    float cmax = -CUDART_INF_F;
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < kDpt; i += 4) {
        const float4 kx = *reinterpret_cast<const float4*>(&ks[j][d0 + i]);
        acc = fmaf(qv[i], kx.x, acc);
        acc = fmaf(qv[i + 1], kx.y, acc);
        acc = fmaf(qv[i + 2], kx.z, acc);
        acc = fmaf(qv[i + 3], kx.w, acc);
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);   // the four slices of the row
      acc += __shfl_xor_sync(0xffffffffu, acc, 2);
      s[j] = (k0 + j <= my_last) ? acc : -CUDART_INF_F;
      cmax = fmaxf(cmax, s[j]);
    }
    const float m_new = fmaxf(m, cmax);
    if (m_new == -CUDART_INF_F) continue;                    // nothing visible yet
    const float corr = exp2f(m - m_new);
    l *= corr;
#pragma unroll
    for (int i = 0; i < kDpt; ++i) o[i] *= corr;
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const float p = exp2f(s[j] - m_new);
      l += p;
#pragma unroll
      for (int i = 0; i < kDpt; i += 4) {
        const float4 vx = *reinterpret_cast<const float4*>(&vs[j][d0 + i]);
        o[i] = fmaf(p, vx.x, o[i]);
        o[i + 1] = fmaf(p, vx.y, o[i + 1]);
        o[i + 2] = fmaf(p, vx.z, o[i + 2]);
        o[i + 3] = fmaf(p, vx.w, o[i + 3]);
      }
    }
    m = m_new;
  }
  if (bad_page && a.status) atomicOr(a.status, kStatusBadPage);
  if (!valid) return;
  const float inv = 1.f / l;
  float4* op = reinterpret_cast<float4*>(a.out + (grow * a.h_q + head) * D + d0);
#pragma unroll
  for (int i = 0; i < kDpt / 4; ++i)
    op[i] = make_float4(o[4 * i] * inv, o[4 * i + 1] * inv, o[4 * i + 2] * inv, o[4 * i + 3] * inv);
  if (sub == 0 && a.lse) a.lse[grow * a.h_q + head] = (m + log2f(l)) * 0.69314718055994531f;
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
  const int64_t grid = n_items * h_q * kRowGroups;
  if (grid == 0) return ZZ_OK;
  if (grid > INT32_MAX) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: grid too large");
  if (d == 64) attn_simt_kernel<64><<<unsigned(grid), kSimtThreads, 0, s>>>(a);
  else attn_simt_kernel<128><<<unsigned(grid), kSimtThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("attn_simt launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}

}  // namespace zz
