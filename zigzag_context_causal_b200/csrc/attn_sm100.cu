// Zigzag prefill attention on the 5th-generation tensor core (sm_100a).
//
// Problem (page "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
// run_attention + build_metadata): for every virtual rank r, half h in
// {prev, next}, sequence s and query head i, causal attention of the half's
// Lq query rows against the first kv_len keys of the sequence; query row j sits
// at position kv_len - Lq + j.  Grouped K/V: query head i reads K/V head
// i / (H_q/H_kv) ("PR #34485 完整报告", implementation item 1).
//
// One CTA owns two 128-row query sub-tiles that stream the SAME K/V tiles:
//   * even GQA group: the same rows of two query heads that share a K/V head
//     (identical causal extent), or
//   * otherwise: two consecutive row tiles of one head (the second one sees
//     one more K/V tile at most).
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax for sub-tile 0   (thread = TMEM lane = query row)
//   warps 4-7  softmax for sub-tile 1
//   warp  8    MMA issue (one thread) + TMEM allocation
//   warp  9    TMA producer: Q once, then K/V stages (V_{j-1}, K_j) into a smem ring
//   warps 10-11 idle
// Launched at 168 registers a thread; the softmax warpgroups grow to 192 and
// the third warpgroup shrinks to 120 (192 + 192 + 120 = 3 x 168 per SM
// sub-partition), so a whole 128-column row of S stays in registers with no
// spills.
// TMEM (512 columns): S0 [0,128)  S1 [128,256)  O0 [256,256+D)  O1 [256+D,256+2D).
// P (bf16, two per column) overwrites the first 64 columns of its S tile and
// feeds the P.V MMA straight from TMEM.  The MMA order per K/V tile j is
//   PV0(j)  S0(j+1)  PV1(j)  S1(j+1)
// so each softmax group works on one tile while the tensor core runs the
// other group's MMAs.  The softmax takes the exact row maximum on a row's
// first tile only and afterwards exponentiates against the running maximum,
// redoing a tile (with O rescaled in TMEM) only when its row sum leaves the
// range (softmax_tile), so the row-maximum pass is off the per-tile chain.
// Tiles past the causal diagonal are never loaded.
//
// attn_fwd_pair (further down) is the same pipeline on clusters of two CTAs
// whose MMAs are shared (tcgen05 .cta_group::2, M = 256), for head_dim 128:
// per SM it loads half the K/V bytes and issues half the TMA boxes, which is
// what bounds small pages.  It is persistent: a cluster that finishes a work
// unit takes the unit of a cluster that has not started yet, by cancelling
// that cluster's launch (cluster launch control), so the next unit's Q load
// and first S overlap the current unit's last P.V and epilogue and no
// cluster pays the barrier/TMEM set-up twice.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <string>
#include <type_traits>

#include "ptx_sm100.cuh"
#include "exp2_poly.h"
#include "nvtx_range.h"
#include "zz_internal.h"

namespace zz {

zz_status_t launch_attn_simt_fp32(const zz_plan_t* p, int rank_begin, int rank_count,
                                  const void* q, const void* k_pool, const void* v_pool,
                                  int64_t num_slots, const int32_t* page_table, int max_pages,
                                  int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                                  float scale, int causal, cudaStream_t s);

namespace {

using namespace zz::dev;

constexpr int kThreads = 384;
constexpr uint32_t kRegsSoftmax = 192, kRegsOther = 120;
constexpr int kWarpMma = 8;
constexpr int kWarpLoad = 9;
constexpr uint32_t kTmemCols = 512;
// Online softmax with a lagging maximum: the row maximum is taken exactly on a
// row's first K/V tile only.  Later tiles use the running maximum m as it is;
// any m at or below the true running maximum gives the same O and l (both
// carry the factor 2^-m), it only has to keep P finite.  The tile's row sum
// bounds every P of the tile, so a tile whose sum exceeds kRedoSum is redone
// against its own maximum after O and l are rescaled.
constexpr float kRedoSum = 65536.0f;   // P <= 2^16 on every tile that is kept
// Bit e of kPolyMask: exponential pair e (of the 16 pairs of each 32-column
// chunk of an S row) is evaluated with the FMA-pipe polynomial of exp2_poly.h
// instead of MUFU ex2, on tiles that need no causal mask (masked tiles keep
// ex2, whose 2^-inf is exactly 0).  Per K/V tile the MUFU work of both
// softmax groups equals the tensor-core work, so moving a share of the
// exponentials to the FMA pipe shortens each sub-tile's softmax.
#ifndef ZZ_POLY_MASK
#define ZZ_POLY_MASK 0u
#endif
constexpr uint32_t kPolyMask = ZZ_POLY_MASK;

template <int D>
struct Cfg {
  static constexpr int kBoxes = D / 64;                  // 128-byte swizzle boxes per row
  static constexpr int kBoxBytes = 128 * 128;            // 128 rows x 128 bytes
  static constexpr int kTileBytes = kBoxes * kBoxBytes;  // one Q, K or V tile
  // K/V ring: stage t holds K_t (second half) and V_{t-1} (first half), the two
  // tiles the MMA issuer consumes in the same iteration.
  static constexpr int kStages = D == 64 ? 4 : 2;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kStageBytes;
  static constexpr int kSmem = kBarOff + 512 + 1024;     // + barriers + alignment slack
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 256 + D;
};

struct Params {
  const HalfDesc* halves;
  const WorkItem* items;
  const int32_t* page_table;
  const __nv_bfloat16* k_pool;
  const __nv_bfloat16* v_pool;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  int64_t num_slots;
  int h_q, h_kv, group;
  int pair_heads;       // 1: sub-tiles are heads 2g, 2g+1; 0: row tiles 2t, 2t+1 of head g
  int head_groups;      // CTAs per work item
  int groups_per_kv;    // head groups that read the same K/V head
  int chunk_items;      // work items per scheduling chunk (see block_coords)
  int n_items;
  int M, rank_begin;
  int max_pages, page_size, box_rows;
  int num_pages;        // ceil(num_slots / page_size): valid page ids are [0, num_pages)
  float scale_log2;
  uint64_t timeout_ns;
  int causal;           // 0: every row of a half sees all kv_full keys of its sequence
  int pair_rows;        // CTA-pair kernel: 1 = four row tiles of one head per cluster, 0 = four heads
};

struct Bars {
  uint64_t q_full[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t mma_done;
  uint64_t kv_full[8];
  uint64_t kv_empty[8];
  uint32_t tmem_base;
  int abort;
  // CTA-pair kernel: the ring that hands each cluster's next work unit to
  // every role of both CTAs, and the cluster-launch-control response.
  uint64_t unit_full[4];
  uint64_t unit_empty[4];   // leader CTA only
  uint64_t clc_full;
  alignas(16) uint32_t clc_resp[4];
  int unit_id[4];
  uint32_t clc_issued;   // cancel requests issued (by the MMA thread)
};

// The unit ring: entry k (slot k % kUnitRing) holds the cluster's (k + 2)-th
// work unit (the first is its own blockIdx), -1 once none is left.  The
// leader's producer writes each entry into both CTAs; every other role of
// both CTAs takes it and frees it with one arrival on the leader's unit_empty.
constexpr int kUnitRing = 4;
// The MMA thread asks for the next unit kClcLead K/V tiles before it issues
// the unit's last S (that is, about kClcLead + 1 tiles before the cluster is
// free): late enough that the hand-out stays dynamic, early enough that the
// answer is there when the producer needs the next Q.
constexpr int kClcLead = 2;
constexpr int kUnitReaders = 18;   // leader: MMA thread + 8 softmax warps; peer: producer + 8 softmax warps

__device__ __forceinline__ bool ring_put(Bars* bars, uint32_t k, int vc, volatile int* abort,
                                         uint64_t timeout_ns) {
  const int slot = int(k % kUnitRing);
  const uint32_t use = k / kUnitRing;
  if (!wait_parity_cluster(&bars->unit_empty[slot], (use & 1u) ^ 1u, abort, timeout_ns)) return false;
  for (uint32_t dst = 0; dst < 2; ++dst) {
    st_cluster_u32(mapa_shared(smem_u32(&bars->unit_id[slot]), dst), uint32_t(vc));
    mbar_arrive_release_cluster(mapa_shared(smem_u32(&bars->unit_full[slot]), dst));
  }
  return true;
}
// Next unit for a reader: the unit index, -1 when none is left, -2 on abort or timeout.
__device__ __forceinline__ int ring_take(Bars* bars, uint32_t lead_unit_empty0, uint32_t k, volatile int* abort,
                                         uint64_t timeout_ns) {
  const int slot = int(k % kUnitRing);
  if (!wait_parity_cluster(&bars->unit_full[slot], (k / kUnitRing) & 1u, abort, timeout_ns)) return -2;
  const int vc = *reinterpret_cast<volatile int*>(&bars->unit_id[slot]);
  mbar_arrive_release_cluster(lead_unit_empty0 + uint32_t(slot) * 8u);
  return vc;
}

static_assert(sizeof(Bars) <= 512, "barrier block of 512 bytes");

struct SubTile {
  int head;
  int q0;   // first half-local row
  int n;    // K/V tiles to visit (0 = empty sub-tile)
};

__device__ __forceinline__ int tiles_for(const HalfDesc& h, int q0, int causal) {
  if (q0 >= h.lq) return 0;
  if (!causal) return (h.kv_full + 127) / 128;
  const int last_row = min(q0 + 128, h.lq) - 1;
  return (h.kv_pos0 + last_row) / 128 + 1;
}

// Softmax of one K/V tile for one query row (thread = TMEM lane): S(j) of the
// row in registers (causal mask applied) -> P = 2^(s*scale*log2e - m) as bf16
// pairs over the first 64 columns of the row's S in TMEM; updates m and l and,
// when a tile is redone, rescales the row's O (D columns at t_o) in TMEM.
// S(j) completing implies P.V(j-1) completed, so O is stable here.  All TMEM
// accesses are warp-wide (.sync.aligned), so every branch around them is
// taken by the whole warp.
template <int D>
__device__ __forceinline__ void softmax_tile(const uint32_t (&sr)[128], int j, bool masked, float scale_log2,
                                             uint32_t t_s, uint32_t t_o, float& m, float& l) {
  auto row_max = [&]() {   // 8 independent max3 chains (short dependency depth)
    float pm[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) pm[q] = fmaxf(__uint_as_float(sr[q]), __uint_as_float(sr[q + 8]));
#pragma unroll
    for (int c = 16; c < 128; c += 16)
#pragma unroll
      for (int q = 0; q < 8; q += 2)
        pm[q] = fmax3(pm[q], __uint_as_float(sr[c + q]), __uint_as_float(sr[c + q + 8])),
        pm[q + 1] = fmax3(pm[q + 1], __uint_as_float(sr[c + q + 1]), __uint_as_float(sr[c + q + 9]));
    return fmaxf(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], fmax3(pm[5], pm[6], pm[7]))) * scale_log2;
  };
  // P of the whole row: packed FMA, ex2 (or the polynomial), packed running
  // sum, bf16 pairs into TMEM.  Returns the tile's row sum.
  auto exp_pass = [&](auto use_poly) {
    const float2 sl2 = make_float2(scale_log2, scale_log2);
    const float2 nm2 = make_float2(-m, -m);
    float2 acc4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                      make_float2(0.f, 0.f)};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int col = c * 32 + 2 * e;
        float2 x = ffma2(make_float2(__uint_as_float(sr[col]), __uint_as_float(sr[col + 1])), sl2, nm2);
        if (decltype(use_poly)::value && ((kPolyMask >> e) & 1u)) {
          x = exp2_poly2(x);
        } else {
          x.x = ex2(x.x);
          x.y = ex2(x.y);
        }
        acc4[e & 3] = fadd2(acc4[e & 3], x);
        pk[e] = pack_bf16x2(x.x, x.y);
      }
      tmem_st16(t_s + c * 16, pk);
    }
    const float2 acc = fadd2(fadd2(acc4[0], acc4[1]), fadd2(acc4[2], acc4[3]));
    return acc.x + acc.y;
  };
  auto exp_any = [&]() {
    return (kPolyMask == 0u || masked) ? exp_pass(std::false_type{}) : exp_pass(std::true_type{});
  };
  if (j == 0) m = row_max();
  float l_tile = exp_any();
  if (j > 0 && __any_sync(0xffffffffu, !(l_tile <= kRedoSum))) {
    // Rows whose maximum did not move keep m (factor exactly 1, same P).
    const float m_new = fmaxf(m, row_max());
    const float f = ex2(m - m_new);
    m = m_new;
    tmem_wait_st();                      // the first pass's P lands before it is overwritten
    l_tile = exp_any();
    l *= f;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(t_o + c * 32, o);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
      tmem_st32(t_o + c * 32, o);
    }
  }
  l += l_tile;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_sm100(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = Cfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work decomposition ----
  // Blocks run in index order.  Items are taken in chunks of chunk_items
  // (longest first); inside a chunk the blocks go K/V head by K/V head, so a
  // wave of resident CTAs is many items x the query heads of ONE K/V head, all
  // streaming the same K/V tiles at about the same time (L2 reuse).
  int item_idx, hg;
  {
    const int per_chunk = p.chunk_items * p.head_groups;
    const int chunk = blockIdx.x / per_chunk;
    const int r = blockIdx.x - chunk * per_chunk;
    const int w_items = min(p.chunk_items, p.n_items - chunk * p.chunk_items);
    const int kvh = r / (w_items * p.groups_per_kv);
    const int r2 = r - kvh * w_items * p.groups_per_kv;
    item_idx = chunk * p.chunk_items + r2 / p.groups_per_kv;
    hg = kvh * p.groups_per_kv + r2 % p.groups_per_kv;
  }
  const WorkItem w = p.items[item_idx];
  const HalfDesc hd = p.halves[w.half_id];
  SubTile st[2];
  if (p.pair_heads) {
    st[0] = {2 * hg, w.tile * 128, 0};
    st[1] = {2 * hg + 1, w.tile * 128, 0};
  } else {
    st[0] = {hg, (2 * w.tile) * 128, 0};
    st[1] = {hg, (2 * w.tile + 1) * 128, 0};
  }
  st[0].n = tiles_for(hd, st[0].q0, p.causal);
  st[1].n = tiles_for(hd, st[1].q0, p.causal);
  const int kv_end = p.causal ? hd.kv_len : hd.kv_full;   // keys that exist for this half
  const int n_max = max(st[0].n, st[1].n);
  const int kv_head = st[0].head / p.group;
  const int64_t row_base = int64_t(hd.rank - p.rank_begin) * p.M + hd.row0;  // Q/O row of half row 0

  // ---- setup ----
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 128);
      mbar_init(&bars->o_full[i], 1);
    }
    mbar_init(&bars->mma_done, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->kv_full[s], 1);
      mbar_init(&bars->kv_empty[s], 1);
    }
    // A CTA that timed out earlier in this launch (or an earlier launch of
    // this plan) has set the status word: skip the work instead of waiting.
    bars->abort = (p.status && (*reinterpret_cast<volatile int*>(p.status) & kStatusTimeout)) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp >= 8) {
  // Third warpgroup: one setmaxnreg for all four warps, then per-warp roles.
  regs_dec<kRegsOther>();
  if (warp == kWarpLoad) {
    // ================= TMA producer =================
    const int32_t* pt = p.page_table + int64_t(hd.seq) * p.max_pages;
    bool q_issued[2] = {false, false};
    if (lane == 0 && !*abort) {
      for (int i = 0; i < 2; ++i) {
        if (st[i].n == 0) continue;
        q_issued[i] = true;
        uint8_t* dst = smem + C::kQOff + i * C::kTileBytes;
        mbar_arrive_expect_tx(&bars->q_full[i], C::kTileBytes);
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(dst + b * C::kBoxBytes, &tm_q, &bars->q_full[i], b * 64, st[i].head,
                      int32_t(row_base + st[i].q0));
      }
    }
    const int chunks = 128 / p.box_rows;
    bool bad_page = false;
    // Stage t (t = 0 .. n_max): K_t if t < n_max, V_{t-1} if t >= 1.
    int t = 0;
    for (; t <= n_max && !*abort; ++t) {
      const int slot = t % C::kStages;
      const uint32_t use = t / C::kStages;
      if (!wait_parity(&bars->kv_empty[slot], (use & 1u) ^ 1u, abort, p.timeout_ns)) break;
      uint8_t* stage = smem + C::kKVOff + slot * C::kStageBytes;
      uint32_t tma_bytes = 0;
      for (int which = 0; which < 2; ++which) {       // 0: V_{t-1} (first half), 1: K_t (second half)
        const int tile_j = which ? t : t - 1;
        if (tile_j < 0 || tile_j >= n_max) continue;
        uint8_t* tile = stage + which * C::kTileBytes;
        const __nv_bfloat16* pool = which ? p.k_pool : p.v_pool;
        const int key0 = tile_j * 128;
        // Rows at or beyond kv_len (end of the sequence's keys) are filled by
        // hand: real keys copied, the rest zero, so no stale or unwritten pool
        // slot can reach the MMAs (0 * NaN would poison P.V).
        bool manual = false;
        for (int c = 0; c < chunks; ++c) {
          if (key0 + (c + 1) * p.box_rows <= kv_end) tma_bytes += p.box_rows * 128 * C::kBoxes;
          else manual = true;
        }
        if (manual) {
          const int units_per_row = C::kBoxes * 8;
          for (int c = 0; c < chunks; ++c) {
            if (key0 + (c + 1) * p.box_rows <= kv_end) continue;
            const int r_lo = c * p.box_rows;
            for (int u = lane; u < p.box_rows * units_per_row; u += 32) {
              const int row = r_lo + u / units_per_row;
              const int rem = u % units_per_row;
              const int b = rem >> 3, ch = rem & 7;
              const int key = key0 + row;
              int4 v = make_int4(0, 0, 0, 0);
              if (key < kv_end) {
                const int64_t slot_id = int64_t(__ldg(pt + key / p.page_size)) * p.page_size + key % p.page_size;
                if (slot_id >= 0 && slot_id < p.num_slots)
                  v = __ldg(reinterpret_cast<const int4*>(pool + (slot_id * p.h_kv + kv_head) * D + b * 64 + ch * 8));
                else
                  bad_page = true;
              }
              *reinterpret_cast<int4*>(tile + b * C::kBoxBytes + row * 128 + ((ch ^ (row & 7)) << 4)) = v;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
        }
      }
      // Lane 0 posts the byte count first; then one lane per page chunk (up to
      // 2 x 16 chunks for 8-token pages) reads its page-table entry and issues
      // that chunk's boxes, so small pages cost one lookup latency per stage.
      if (lane == 0) mbar_arrive_expect_tx(&bars->kv_full[slot], tma_bytes);
      __syncwarp();
      for (int u = lane; u < 2 * chunks; u += 32) {
        const int which = u / chunks, c = u - which * chunks;
        const int tile_j = which ? t : t - 1;
        if (tile_j < 0 || tile_j >= n_max) continue;
        const int kc = tile_j * 128 + c * p.box_rows;
        if (kc + p.box_rows > kv_end) continue;
        uint8_t* tile = stage + which * C::kTileBytes;
        const void* tm = which ? static_cast<const void*>(&tm_k) : static_cast<const void*>(&tm_v);
        // A page outside the pool is loaded from a coordinate past the pool's
        // end (zero fill) and reported through the status word.
        const int32_t page = __ldg(pt + kc / p.page_size);
        const bool in_pool = uint32_t(page) < uint32_t(p.num_pages);
        bad_page |= !in_pool;
        const int32_t slot0 = (in_pool ? page : p.num_pages) * p.page_size + kc % p.page_size;
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(tile + b * C::kBoxBytes + c * p.box_rows * 128, tm, &bars->kv_full[slot],
                      b * 64, kv_head, slot0);
      }
      __syncwarp();
    }
    const int load_no = t;   // stages issued
    if (bad_page && p.status) atomicOr(p.status, kStatusBadPage);
    // Never leave with copies in flight into shared memory.
    if (lane == 0) {
      for (int n = max(0, load_no - C::kStages); n < load_no; ++n)
        drain_parity(&bars->kv_full[n % C::kStages], (uint32_t(n / C::kStages)) & 1u, p.timeout_ns);
      for (int i = 0; i < 2; ++i)
        if (q_issued[i]) drain_parity(&bars->q_full[i], 0, p.timeout_ns);
    }
  } else if (warp == kWarpMma) {
    // ================= MMA issue (single thread) =================
    // A single thread retires a tcgen05.mma only every ~50 cycles, little faster
    // than a 128x128x16 MMA executes (64 cycles), so everything else this thread
    // does between MMAs (barrier waits, commits) must stay short: descriptors
    // are a base plus a compile-time offset, the sub-tile code is unrolled, and
    // each K/V tile costs one full-wait and one release (stage = V_j + K_{j+1}).
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t kv_addr = smem_u32(smem + C::kKVOff);
      // K-major operands (Q, K): SBO = 8 rows x 128 B; MN-major V: LBO = next 64-column box.
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
      const uint64_t dq1 = dq0 + uint64_t(C::kTileBytes >> 4);
      const uint64_t dk0 = smem_desc_sw128(kv_addr + C::kTileBytes, 16, 1024);   // K half of stage 0
      const uint64_t dv0 = smem_desc_sw128(kv_addr, C::kBoxBytes, 1024);         // V half of stage 0
      const int n0 = st[0].n, n1 = st[1].n;
      auto issue_s = [&](uint32_t col, uint64_t dq, int slot) {
        const uint64_t dk = dk0 + uint64_t((slot * C::kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = uint64_t(((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4);
          mma_ss(tmem + col, dq + off, dk + off, idesc_s, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t col_o, uint32_t col_p, int slot, bool acc) {
        const uint64_t dv = dv0 + uint64_t((slot * C::kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts(tmem + col_o, tmem + col_p + kk * 8, dv + uint64_t((kk * 2048) >> 4), idesc_o,
                 (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = true;
      if (n0) ok = wait_parity(&bars->q_full[0], 0, abort, p.timeout_ns);
      if (ok && n1) ok = wait_parity(&bars->q_full[1], 0, abort, p.timeout_ns);
      if (ok) ok = wait_parity(&bars->kv_full[0], 0, abort, p.timeout_ns);   // stage 0: K_0
      if (ok) {
        tc_fence_after();
        if (n0) { issue_s(C::kColS0, dq0, 0); mma_commit(&bars->s_full[0]); }
        if (n1) { issue_s(C::kColS1, dq1, 0); mma_commit(&bars->s_full[1]); }
        mma_commit(&bars->kv_empty[0]);
      }
      for (int j = 0; j < n_max && ok; ++j) {
        const int t = j + 1;                    // stage with V_j and K_{j+1}
        const int slot = t % C::kStages;
        if (!(ok = wait_parity(&bars->kv_full[slot], uint32_t(t / C::kStages) & 1u, abort, p.timeout_ns))) break;
        if (j < n0) {
          if (!(ok = wait_spin(&bars->p_full[0], uint32_t(j) & 1u, abort, p.timeout_ns))) break;
          tc_fence_after();
          issue_pv(C::kColO0, C::kColS0, slot, j > 0);
          if (j == n0 - 1) mma_commit(&bars->o_full[0]);
          else { issue_s(C::kColS0, dq0, slot); mma_commit(&bars->s_full[0]); }
        }
        if (j < n1) {
          if (!(ok = wait_spin(&bars->p_full[1], uint32_t(j) & 1u, abort, p.timeout_ns))) break;
          tc_fence_after();
          issue_pv(C::kColO1, C::kColS1, slot, j > 0);
          if (j == n1 - 1) mma_commit(&bars->o_full[1]);
          else { issue_s(C::kColS1, dq1, slot); mma_commit(&bars->s_full[1]); }
        }
        mma_commit(&bars->kv_empty[slot]);
      }
      // Drain: no MMA may still be running when TMEM is released.
      mma_commit(&bars->mma_done);
      drain_parity(&bars->mma_done, 0, p.timeout_ns);
    }
    __syncwarp();
  }   // warps 10-11 have no role
  } else {
    // ================= softmax + epilogue (warps 0-7) =================
    regs_inc<kRegsSoftmax>();
    const int g = warp >> 2;                   // sub-tile
    const SubTile& me = st[g];
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;         // TMEM lane == row of the sub-tile
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + (g ? C::kColS1 : C::kColS0);
    const uint32_t t_o = tmem + lane_off + (g ? C::kColO1 : C::kColO0);
    const int q_row = me.q0 + r;
    // Last visible key (inclusive) of my row and of the sub-tile's first row;
    // without the causal mask every row sees the whole sequence.
    const int my_pos = p.causal ? hd.kv_pos0 + q_row : hd.kv_full - 1;
    const int first_pos = p.causal ? hd.kv_pos0 + me.q0 : hd.kv_full - 1;
    float m = -CUDART_INF_F, l = 0.f;
    bool ok = me.n > 0;
    for (int j = 0; j < me.n && ok; ++j) {
      ok = wait_parity(&bars->s_full[g], uint32_t(j) & 1u, abort, p.timeout_ns);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }   // TMEM access below is warp-wide
      tc_fence_after();
      // The whole 128-column row of S in registers: four loads, one wait.
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      // Causal mask, only on tiles that reach past the sub-tile's first row.
      const bool masked = j * 128 + 127 > first_pos;
      if (masked) {
        const int limit = my_pos - j * 128 + 1;   // visible keys of this row in this tile
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= limit) sr[c] = 0xFF800000u;     // -inf
      }
      softmax_tile<D>(sr, j, masked, p.scale_log2, t_s, t_o, m, l);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[g]);
    }
    if (ok) ok = wait_parity(&bars->o_full[g], 0, abort, p.timeout_ns);
    ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-wide
    if (ok) {
      tc_fence_after();
      const bool valid = q_row < hd.lq;
      const int64_t grow = row_base + q_row;
      const float inv = 1.f / l;
      __nv_bfloat16* op = p.out + (grow * p.h_q + me.head) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(t_o + c * 32, o);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
        if (valid) {
          int4* dst = reinterpret_cast<int4*>(op + c * 32);
#pragma unroll
          for (int v = 0; v < 4; ++v)
            dst[v] = make_int4(int(pk[4 * v]), int(pk[4 * v + 1]), int(pk[4 * v + 2]), int(pk[4 * v + 3]));
        }
      }
      if (valid && p.lse) p.lse[grow * p.h_q + me.head] = (m + log2f(l)) * 0.69314718055994531f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort && p.status) {
    atomicOr(p.status, kStatusTimeout);
    __threadfence();
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
// attn_fwd_pair: the same attention with two CTAs per MMA (tcgen05 .cta_group::2),
// for D = 128.  A cluster of two CTAs takes four 128-row sub-tiles that share a
// K/V head: with a GQA group that is a multiple of 4, the same row tile of four
// query heads (CTA rank r owns heads 4u + 2r and 4u + 2r + 1); otherwise four
// consecutive row tiles of one head (CTA rank r owns tiles 4t + 2r and
// 4t + 2r + 1), all run to the keys of the last one.  Each pair MMA
// has M = 256 (128 rows from each CTA) and splits B by N across the pair, so
// every CTA loads only half of each K tile (64 keys, all 128 dims) and half of
// each V tile (all 128 keys, 64 dims): per SM, half the K/V bytes and half the
// TMA boxes of the single-CTA kernel for the same FLOPs.  CTA 0 issues every
// MMA; its commits arrive on the barriers of both CTAs.
struct PairCfg {
  static constexpr int kBoxBytes = 128 * 128;
  static constexpr int kQBytes = 2 * kBoxBytes;           // Q tile: 128 rows x 128 dims
  static constexpr int kKHalfBytes = 2 * 64 * 128;        // 64 keys x 128 dims (two 8 KB column boxes)
  static constexpr int kVHalfBytes = 128 * 128;           // 128 keys x 64 dims (one box)
  static constexpr int kStageBytes = kKHalfBytes + kVHalfBytes;
  static constexpr int kStages = 5;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kQBytes;
  static constexpr int kBarOff = kKVOff + kStages * kStageBytes;
  static constexpr int kSmem = kBarOff + 512 + 1024;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
};
static_assert(PairCfg::kSmem <= 232448, "227 KB of shared memory per CTA");
// setmaxnreg split of the pair kernel (the one without spills for its code).
constexpr uint32_t kPairRegsSoftmax = 192, kPairRegsOther = 120;
static_assert(2 * kPairRegsSoftmax + kPairRegsOther <= 3 * 168, "register split exceeds the launch's registers");

// One work unit of the pair kernel (one cluster of the grid): unit index vc ->
// work item, this CTA's two sub-tiles and the K/V range they share.  Units are
// numbered in chunks of work items (longest first), K/V-head-major inside a
// chunk, so that clusters running at the same time stream the same K/V tiles
// through L2.
// Heads mode (GQA group a multiple of 4): a unit is a quad of query heads of
// one K/V head and one row tile; CTA rank r takes heads 4u + 2r, 4u + 2r + 1.
// Rows mode (any other group): a unit is one query head and a quad of row
// tiles; CTA rank r takes row tiles 4t + 2r and 4t + 2r + 1.
struct PairUnit {
  HalfDesc hd;
  SubTile st[2];
  int n;              // K/V tiles every sub-tile of the unit visits (they share each MMA)
  int kv_end, kv_head;
  int64_t row_base;   // Q/O row of the half's row 0
};

__device__ __forceinline__ PairUnit pair_unit(const Params& p, int vc, uint32_t rank) {
  const int units_per_kv = p.pair_rows ? p.group : (p.groups_per_kv >> 1);
  const int per_chunk = p.chunk_items * (p.pair_rows ? p.h_q : (p.head_groups >> 1));
  const int chunk = vc / per_chunk;
  const int r = vc - chunk * per_chunk;
  const int w_items = min(p.chunk_items, p.n_items - chunk * p.chunk_items);
  const int kvh = r / (w_items * units_per_kv);
  const int r2 = r - kvh * w_items * units_per_kv;
  const int item_idx = chunk * p.chunk_items + r2 / units_per_kv;
  const int unit = kvh * units_per_kv + r2 % units_per_kv;
  const WorkItem w = p.items[item_idx];
  PairUnit u;
  u.hd = p.halves[w.half_id];
  if (p.pair_rows) {
    u.st[0] = {unit, (4 * w.tile + 2 * int(rank)) * 128, 0};
    u.st[1] = {unit, (4 * w.tile + 2 * int(rank) + 1) * 128, 0};
    // the keys of the quad's last valid row tile; lower rows see the extra
    // tiles fully masked (P = 0), rows past the half are computed and not written
    const int last_tile = min(4 * w.tile + 3, (u.hd.lq - 1) / 128);
    u.n = tiles_for(u.hd, last_tile * 128, p.causal);
  } else {
    u.st[0] = {4 * unit + 2 * int(rank), w.tile * 128, 0};
    u.st[1] = {4 * unit + 2 * int(rank) + 1, w.tile * 128, 0};
    u.n = tiles_for(u.hd, u.st[0].q0, p.causal);          // same rows, same keys
  }
  u.st[0].n = u.n;
  u.st[1].n = u.n;
  u.kv_end = p.causal ? u.hd.kv_len : u.hd.kv_full;
  u.kv_head = u.st[0].head / p.group;
  u.row_base = int64_t(u.hd.rank - p.rank_begin) * p.M + u.hd.row0;
  return u;
}

// Persistent over units: a cluster does the unit of its own blockIdx, then
// takes the units of clusters that have not started yet (cluster launch
// control cancels their launch), until none is left.  The MMA thread asks for
// the next unit a few tiles before the end of the current one; the leader's
// producer reads the answer and hands it to every role through the unit ring.
// All roles walk the same unit sequence, so the barrier phases carry over from
// unit to unit (per-role counts of units, K/V stages and tiles).  Once the
// producer has issued the current unit's stages it already loads the next
// unit's first K/V stages into the slots the MMA frees, and the next unit's Q
// as soon as the current unit's last S MMAs have read Q (q_free); the next
// unit's first S then runs while the current unit's last P.V and epilogue do.
// Every planned unit has rows (the planner emits only row tiles that start
// inside their half), so n >= 1 for every unit; the producer relies on it.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
attn_fwd_pair(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const Params p) {
  using C = PairCfg;
  constexpr int D = 128;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();     // 0: leader (issues the MMAs), 1: peer
  const bool leader = rank == 0;
  const int vc0 = int(blockIdx.x >> 1);        // the cluster's first unit

  // ---- setup: barriers in both CTAs, TMEM for the pair, then a cluster barrier
  // so that no CTA signals the other's barriers before they exist ----
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full[0], 2);        // one expect_tx arrival from each CTA's producer (both Q tiles)
    mbar_init(&bars->q_full[1], 1);        // q_free: the unit's last S MMAs have read Q (commit)
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->p_full[i], 256);    // 128 softmax threads of each CTA
      mbar_init(&bars->o_full[i], 1);
    }
    mbar_init(&bars->mma_done, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->kv_full[s], 2);     // one expect_tx arrival from each CTA's producer
      mbar_init(&bars->kv_empty[s], 1);
    }
    for (int i = 0; i < kUnitRing; ++i) {
      mbar_init(&bars->unit_full[i], 1);
      mbar_init(&bars->unit_empty[i], kUnitReaders);
    }
    mbar_init(&bars->clc_full, 1);
    bars->clc_issued = 0;
    bars->abort = (p.status && (*reinterpret_cast<volatile int*>(p.status) & kStatusTimeout)) ? 1 : 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc_pair(&bars->tmem_base, kTmemCols);
    tmem_relinquish_pair();
    tc_fence_before();
  }
  if (warp == kWarpLoad && lane == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  uint64_t* q_full = &bars->q_full[0];
  uint64_t* q_free = &bars->q_full[1];
  // The leader's barriers, as shared::cluster addresses (the peer signals them remotely).
  const uint32_t lead_q_full = mapa_shared(smem_u32(q_full), 0);
  const uint32_t lead_kv_full0 = mapa_shared(smem_u32(&bars->kv_full[0]), 0);
  const uint32_t lead_p_full0 = mapa_shared(smem_u32(&bars->p_full[0]), 0);
  const uint32_t lead_unit_empty0 = mapa_shared(smem_u32(&bars->unit_empty[0]), 0);
  uint32_t clc_read = 0;   // cancel responses read (the leader's producer)

  if (warp >= 8) {
  regs_dec<kPairRegsOther>();
  if (warp == kWarpLoad) {
    // ================= TMA producer (both CTAs: this CTA's halves) =================
    const int kbox = p.box_rows < 64 ? p.box_rows : 64;       // K half: 64 keys
    const int vbox = p.box_rows;                              // V half: 128 keys
    const int kchunks = 64 / kbox, vchunks = 128 / vbox;
    bool bad_page = false;
    int tg = 0;               // K/V stages issued so far (all units)
    uint32_t qk = 0;          // units whose Q was issued
    uint32_t ring_k = 0;      // unit-ring entries written (leader) or taken (peer)
    uint32_t clc_ph = 0;      // phase of clc_full
    uint32_t clc_taken = 0;   // cancel responses read
    // Stage t of unit u (t = 0 .. n) into ring slot `slot`: this CTA's half of
    // K_t if t < n, of V_{t-1} if t >= 1 (the slot is free: kv_empty passed).
    auto issue_stage = [&](const PairUnit& u, const int32_t* pt, int t, int slot) {
      uint8_t* stage = smem + C::kKVOff + slot * C::kStageBytes;
      uint8_t* ktile = stage;
      uint8_t* vtile = stage + C::kKHalfBytes;
      const bool has_k = t < u.n, has_v = t >= 1;
      const int key0k = t * 128 + 64 * int(rank);           // first key of this CTA's K half
      const int key0v = (t - 1) * 128;                       // first key of the V tile
      uint32_t tma_bytes = 0;
      bool manual = false;
      if (has_k)
        for (int c = 0; c < kchunks; ++c) {
          if (key0k + (c + 1) * kbox <= u.kv_end) tma_bytes += kbox * 128 * 2;
          else manual = true;
        }
      if (has_v)
        for (int c = 0; c < vchunks; ++c) {
          if (key0v + (c + 1) * vbox <= u.kv_end) tma_bytes += vbox * 128;
          else manual = true;
        }
      if (manual) {
        // Rows at or beyond kv_len are filled by hand (real keys copied, the rest zero).
        for (int which = 0; which < 2; ++which) {
          if (which == 0 && !has_k) continue;
          if (which == 1 && !has_v) continue;
          const int rows = which == 0 ? 64 : 128, box = which == 0 ? kbox : vbox;
          const int units_per_row = which == 0 ? 16 : 8;   // 16-byte pieces of this CTA's part of a row
          const int key0 = which == 0 ? key0k : key0v;
          const __nv_bfloat16* pool = which == 0 ? p.k_pool : p.v_pool;
          for (int c = 0; c < rows / box; ++c) {
            if (key0 + (c + 1) * box <= u.kv_end) continue;
            for (int e = lane; e < box * units_per_row; e += 32) {
              const int row = c * box + e / units_per_row;
              const int rem = e % units_per_row;
              const int b = rem >> 3, ch = rem & 7;        // column box (K only) and 16-byte piece
              const int key = key0 + row;
              const int col = which == 0 ? b * 64 + ch * 8 : 64 * int(rank) + ch * 8;
              int4 v = make_int4(0, 0, 0, 0);
              if (key < u.kv_end) {
                const int64_t slot_id =
                    int64_t(__ldg(pt + key / p.page_size)) * p.page_size + key % p.page_size;
                if (slot_id >= 0 && slot_id < p.num_slots)
                  v = __ldg(reinterpret_cast<const int4*>(pool + (slot_id * p.h_kv + u.kv_head) * D + col));
                else
                  bad_page = true;
              }
              uint8_t* dstp = which == 0 ? ktile + b * (64 * 128) : vtile;
              *reinterpret_cast<int4*>(dstp + row * 128 + ((ch ^ (row & 7)) << 4)) = v;
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
      }
      const uint32_t bar = lead_kv_full0 + uint32_t(slot) * 8u;
      if (lane == 0) mbar_arrive_expect_tx_cluster(bar, tma_bytes);
      __syncwarp();
      // One lane per page chunk: K chunks first, then V chunks.
      const int nk = has_k ? kchunks : 0, nv = has_v ? vchunks : 0;
      for (int e = lane; e < nk + nv; e += 32) {
        const bool is_k = e < nk;
        const int c = is_k ? e : e - nk;
        const int box = is_k ? kbox : vbox;
        const int kc = (is_k ? key0k : key0v) + c * box;
        if (kc + box > u.kv_end) continue;
        const int32_t page = __ldg(pt + kc / p.page_size);
        const bool in_pool = uint32_t(page) < uint32_t(p.num_pages);
        bad_page |= !in_pool;
        const int32_t slot0 = (in_pool ? page : p.num_pages) * p.page_size + kc % p.page_size;
        if (is_k) {
          for (int b = 0; b < 2; ++b)
            tma_load_3d_pair(ktile + b * (64 * 128) + c * box * 128, &tm_k, bar, b * 64, u.kv_head, slot0);
        } else {
          tma_load_3d_pair(vtile + c * box * 128, &tm_v, bar, 64 * int(rank), u.kv_head, slot0);
        }
      }
      __syncwarp();
    };
    // Q of both sub-tiles of unit u (the previous unit's last S MMAs have read the old Q).
    auto load_q = [&](const PairUnit& u) {
      if (lane == 0) {
        mbar_arrive_expect_tx_cluster(lead_q_full, 2 * C::kQBytes);
        for (int i = 0; i < 2; ++i)
          for (int b = 0; b < 2; ++b)
            tma_load_3d_pair(smem + C::kQOff + i * C::kQBytes + b * C::kBoxBytes, &tm_q, lead_q_full, b * 64,
                             u.st[i].head, int32_t(u.row_base + u.st[i].q0));
      }
      __syncwarp();
    };
    PairUnit u = pair_unit(p, vc0, rank);
    const int32_t* pt = p.page_table + int64_t(u.hd.seq) * p.max_pages;
    int t_next = 0;           // next stage of u to issue
    bool ok = !__any_sync(0xffffffffu, *abort != 0);
    if (ok) { load_q(u); ++qk; }
    while (ok) {
      // The rest of this unit's stages.
      for (; t_next <= u.n; ++t_next, ++tg) {
        const int slot = tg % C::kStages;
        ok = __all_sync(0xffffffffu,
                        wait_parity(&bars->kv_empty[slot], ((tg / C::kStages) & 1u) ^ 1u, abort, p.timeout_ns));
        if (!ok) break;
        issue_stage(u, pt, t_next, slot);
      }
      if (!ok) break;
      // The next unit: the leader reads the answer to the MMA thread's cancel
      // request and hands it on, the peer takes it from the ring.
      int nxt = -2;
      if (lane == 0) {
        if (leader) {
          if (wait_parity(&bars->clc_full, clc_ph, abort, p.timeout_ns)) {
            clc_ph ^= 1u;
            ++clc_taken;
            const int x = clc_first_ctaid_x(bars->clc_resp);
            fence_proxy_async_smem();          // the next response is written through the async proxy
            nxt = x < 0 ? -1 : (x >> 1);
            if (!ring_put(bars, ring_k++, nxt, abort, p.timeout_ns)) nxt = -2;
          }
        } else {
          nxt = ring_take(bars, lead_unit_empty0, ring_k++, abort, p.timeout_ns);
        }
      }
      const int vn = __shfl_sync(0xffffffffu, nxt, 0);
      if (vn < 0) break;
      const PairUnit un = pair_unit(p, vn, rank);
      const int32_t* pt_n = p.page_table + int64_t(un.hd.seq) * p.max_pages;
      // While this unit's last S still reads Q, load the next unit's first
      // K/V stages into the slots the MMA frees; then its Q.
      int tn = 0;
      const uint32_t qf_par = (qk - 1) & 1u;
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 0; tn <= un.n; ++it) {
        if (__shfl_sync(0xffffffffu, mbar_test_wait(q_free, qf_par) ? 1 : 0, 0)) break;
        const int slot = tg % C::kStages;
        if (__shfl_sync(0xffffffffu, mbar_test_wait(&bars->kv_empty[slot], ((tg / C::kStages) & 1u) ^ 1u) ? 1 : 0,
                        0)) {
          issue_stage(un, pt_n, tn, slot);
          ++tn;
          ++tg;
          continue;
        }
        if ((it & 255u) == 255u &&
            __shfl_sync(0xffffffffu, (*abort != 0 || global_timer_ns() - t0 > p.timeout_ns) ? 1 : 0, 0))
          break;   // the blocking wait below gives up the same way
      }
      ok = __all_sync(0xffffffffu, wait_parity(q_free, qf_par, abort, p.timeout_ns));
      if (!ok) break;
      load_q(un);
      ++qk;
      u = un;
      pt = pt_n;
      t_next = tn;
    }
    if (bad_page && p.status) atomicOr(p.status, kStatusBadPage);
    // Copies of both CTAs land on the leader's barriers: the leader's producer
    // drains them; the cluster barrier at the end keeps the peer alive until then.
    if (lane == 0 && leader) {
      for (int k = max(0, tg - C::kStages); k < tg; ++k)
        drain_parity(&bars->kv_full[k % C::kStages], (uint32_t(k / C::kStages)) & 1u, p.timeout_ns);
      if (qk > 0) drain_parity(q_full, (qk - 1) & 1u, p.timeout_ns);
    }
    clc_read = clc_taken;
  } else if (warp == kWarpMma && leader) {
    // ================= MMA issue (leader CTA, one thread) =================
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(256, 128, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(256, D, false, true);
      const uint32_t kv_addr = smem_u32(smem + C::kKVOff);
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + C::kQOff), 16, 1024);
      const uint64_t dq1 = dq0 + uint64_t(C::kQBytes >> 4);
      const uint64_t dk0 = smem_desc_sw128(kv_addr, 16, 1024);                       // K half of stage 0
      const uint64_t dv0 = smem_desc_sw128(kv_addr + C::kKHalfBytes, 16, 1024);      // V half of stage 0
      const uint16_t both = 3;
      auto issue_s = [&](uint32_t col, uint64_t dq, int slot) {
        const uint64_t dk = dk0 + uint64_t((slot * C::kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qoff = ((kk >> 2) * C::kBoxBytes + (kk & 3) * 32) >> 4;
          const uint32_t koff = ((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4;
          mma_ss_pair(tmem + col, dq + qoff, dk + koff, idesc_s, kk > 0);
        }
      };
      auto issue_pv = [&](uint32_t col_o, uint32_t col_p, int slot, bool acc) {
        const uint64_t dv = dv0 + uint64_t((slot * C::kStageBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          mma_ts_pair(tmem + col_o, tmem + col_p + kk * 8, dv + uint64_t((kk * 2048) >> 4), idesc_o,
                      (acc || kk > 0) ? 1u : 0u);
      };
      int tg = 0;            // K/V stages consumed so far (all units)
      uint32_t qk = 0;       // units started
      uint32_t jg = 0;       // tiles of all earlier units (phase base of p_full)
      uint32_t ring_k = 0;   // unit-ring entries taken
      uint32_t issued = 0;   // cancel requests issued
      auto request_next = [&]() {
        mbar_arrive_expect_tx(&bars->clc_full, 16);
        clc_try_cancel(bars->clc_resp, &bars->clc_full);
        ++issued;
      };
      bool ok = true;
      for (int vc = vc0; vc >= 0 && ok;) {
        const int n = pair_unit(p, vc, 0).n;
        const int req_j = n - 2 - kClcLead;   // loop iteration after which to ask (-1: after the first S)
        if (n <= 0) request_next();
        if (n > 0) {
          if (!(ok = wait_parity(q_full, qk & 1u, abort, p.timeout_ns))) break;
          {
            const int slot = tg % C::kStages;                 // stage 0 of the unit: K_0
            if (!(ok = wait_parity(&bars->kv_full[slot], uint32_t(tg / C::kStages) & 1u, abort, p.timeout_ns)))
              break;
            tc_fence_after();
            issue_s(C::kColS0, dq0, slot); mma_commit_pair(&bars->s_full[0], both);
            issue_s(C::kColS1, dq1, slot); mma_commit_pair(&bars->s_full[1], both);
            if (n == 1) mma_commit_pair(q_free, both);        // the unit's last S
            mma_commit_pair(&bars->kv_empty[slot], both);
            ++tg;
            if (req_j < 0) request_next();
          }
          for (int j = 0; j < n && ok; ++j, ++tg) {
            const int slot = tg % C::kStages;                 // stage with V_j and K_{j+1}
            const uint32_t ph = (jg + uint32_t(j)) & 1u;
            if (!(ok = wait_parity(&bars->kv_full[slot], uint32_t(tg / C::kStages) & 1u, abort, p.timeout_ns)))
              break;
            if (!(ok = wait_spin(&bars->p_full[0], ph, abort, p.timeout_ns))) break;
            tc_fence_after();
            issue_pv(C::kColO0, C::kColS0, slot, j > 0);
            if (j == n - 1) mma_commit_pair(&bars->o_full[0], both);
            else { issue_s(C::kColS0, dq0, slot); mma_commit_pair(&bars->s_full[0], both); }
            if (!(ok = wait_spin(&bars->p_full[1], ph, abort, p.timeout_ns))) break;
            tc_fence_after();
            issue_pv(C::kColO1, C::kColS1, slot, j > 0);
            if (j == n - 1) mma_commit_pair(&bars->o_full[1], both);
            else { issue_s(C::kColS1, dq1, slot); mma_commit_pair(&bars->s_full[1], both); }
            if (j == n - 2) mma_commit_pair(q_free, both);    // the unit's last S
            mma_commit_pair(&bars->kv_empty[slot], both);
            if (j == req_j) request_next();
          }
          jg += uint32_t(n);
          ++qk;
        }
        if (ok) vc = ring_take(bars, lead_unit_empty0, ring_k++, abort, p.timeout_ns);
      }
      bars->clc_issued = issued;
      mma_commit_pair(&bars->mma_done, 1);
      drain_parity(&bars->mma_done, 0, p.timeout_ns);
    }
    __syncwarp();
  }   // the peer's MMA warp and warps 10-11 have no role here
  } else {
    // ================= softmax + epilogue (warps 0-7, both CTAs) =================
    regs_inc<kPairRegsSoftmax>();
    const int g = warp >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = uint32_t(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off + (g ? C::kColS1 : C::kColS0);
    const uint32_t t_o = tmem + lane_off + (g ? C::kColO1 : C::kColO0);
    const uint32_t p_full_lead = lead_p_full0 + uint32_t(g) * 8u;
    uint32_t qk = 0;       // units done
    uint32_t jg = 0;       // tiles of all earlier units
    uint32_t ring_k = 0;   // unit-ring entries taken
    int vc = vc0;
    while (vc >= 0) {
      const PairUnit u = pair_unit(p, vc, rank);
      const int my_head = g ? u.st[1].head : u.st[0].head;   // no dynamic index: u stays in registers
      const int my_q0 = g ? u.st[1].q0 : u.st[0].q0;
      const int n = u.n;
      if (n > 0) {
        const int q_row = my_q0 + r;
        const int my_pos = p.causal ? u.hd.kv_pos0 + q_row : u.hd.kv_full - 1;
        const int first_pos = p.causal ? u.hd.kv_pos0 + my_q0 : u.hd.kv_full - 1;
        float m = -CUDART_INF_F, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n && ok; ++j) {
          ok = wait_parity(&bars->s_full[g], (jg + uint32_t(j)) & 1u, abort, p.timeout_ns);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }   // TMEM access below is warp-wide
          tc_fence_after();
          uint32_t sr[128];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          tmem_wait_ld();
          const bool masked = j * 128 + 127 > first_pos;
          if (masked) {
            const int limit = my_pos - j * 128 + 1;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= limit) sr[c] = 0xFF800000u;
          }
          softmax_tile<D>(sr, j, masked, p.scale_log2, t_s, t_o, m, l);
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive_cluster(p_full_lead);       // the leader's barrier, from either CTA
        }
        if (ok) ok = wait_parity(&bars->o_full[g], qk & 1u, abort, p.timeout_ns);
        if (!__all_sync(0xffffffffu, ok)) break;  // the TMEM loads below are warp-wide
        // Epilogue.  Its TMEM loads complete (wait::ld) before this warp writes
        // the next unit's P, so the next unit's first P.V (which overwrites O)
        // cannot race them.
        tc_fence_after();
        const bool valid = q_row < u.hd.lq;
        const int64_t grow = u.row_base + q_row;
        const float inv = 1.f / l;
        __nv_bfloat16* op = p.out + (grow * p.h_q + my_head) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
          tmem_wait_ld();
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(o[2 * e]) * inv, __uint_as_float(o[2 * e + 1]) * inv);
          if (valid) {
            int4* dst = reinterpret_cast<int4*>(op + c * 32);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_int4(int(pk[4 * v]), int(pk[4 * v + 1]), int(pk[4 * v + 2]), int(pk[4 * v + 3]));
          }
        }
        if (valid && p.lse) p.lse[grow * p.h_q + my_head] = (m + log2f(l)) * 0.69314718055994531f;
        jg += uint32_t(n);
        ++qk;
      }
      int nxt = -2;
      if (lane == 0) nxt = ring_take(bars, lead_unit_empty0, ring_k++, abort, p.timeout_ns);
      vc = __shfl_sync(0xffffffffu, nxt, 0);
    }
  }

  // ---- teardown: both CTAs done with TMEM and with each other's barriers ----
  tc_fence_before();
  __syncthreads();
  // A cancel response still in flight (only after an abort: one request at
  // most is outstanding) lands before this CTA's shared memory is released.
  if (leader && warp == kWarpLoad && lane == 0 && bars->clc_issued > clc_read)
    drain_parity(&bars->clc_full, clc_read & 1u, p.timeout_ns);
  cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
  if (threadIdx.x == 0 && bars->abort && p.status) {
    atomicOr(p.status, kStatusTimeout);
    __threadfence();
  }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

zz_status_t get_encoder() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q{};
    void* fn = nullptr;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode)
    return fail(ZZ_ERR_CUDA, std::string("cuTensorMapEncodeTiled unavailable: ") + cudaGetErrorString(err));
  return ZZ_OK;
}

// 3-D bf16 tensor [rows][heads][d] seen as (d, heads, rows); box (64, 1, box_rows), 128B swizzle.
zz_status_t encode_3d(CUtensorMap* m, const void* base, int d, int heads, int64_t rows, int box_rows) {
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(heads), cuuint64_t(rows)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(d) * heads * 2};
  cuuint32_t box[3] = {64, 1, cuuint32_t(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ZZ_ERR_CUDA, "cuTensorMapEncodeTiled failed (" + std::to_string(int(r)) + ")");
  return ZZ_OK;
}

// Items per scheduling chunk: enough that one K/V head's blocks of a chunk
// fill every SM once (one resident CTA per SM).
int chunk_items_for(int groups_per_kv) {
  return std::max(1, (device_sm_count() + groups_per_kv - 1) / groups_per_kv);
}

// The kernel needs more than 48 KB of dynamic shared memory, which must be
// opted into once per function and device (the attribute belongs to the
// device's context); remembered per device ordinal, guarded for host threads.
constexpr int kMaxDevices = 256;
std::mutex g_attr_mu;
bool g_attr_done[kMaxDevices][2] = {};

template <int D>
zz_status_t ensure_smem_attr() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(ZZ_ERR_UNSUPPORTED, "device ordinal above 255");
  std::lock_guard<std::mutex> lock(g_attr_mu);
  bool& done = g_attr_done[dev][D == 128 ? 1 : 0];
  if (!done) {
    e = cudaFuncSetAttribute(attn_fwd_sm100<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<D>::kSmem);
    if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    done = true;
  }
  return ZZ_OK;
}

// Which bf16 kernel a launch runs.  head_dim 128 runs on CTA pairs: four query
// heads of one K/V head per cluster when the GQA group is a multiple of 4,
// otherwise four row tiles of one head.  head_dim 64 runs on single CTAs.
enum KernelChoice { kSingleCta = 0, kPairHeads = 1, kPairRows = 2 };
KernelChoice kernel_for(int d, int group) {
  if (d != 128) return kSingleCta;
  return group % 4 == 0 ? kPairHeads : kPairRows;
}

// The plan's work list for a launch of ranks [rank_begin, rank_begin + rank_count):
// row tiles (head pairs / head quads), row-tile pairs (single CTA, odd groups)
// or row-tile quads (CTA pairs, rows mode).
struct ItemRange {
  const std::vector<WorkItem>* list;   // host copy
  size_t ws_off;                       // its section in the plan workspace
  size_t first, n;                     // first item and item count of the launch
};
ItemRange items_for(const zz_plan_t* pl, KernelChoice k, bool pair_heads, int rank_begin, int rank_count) {
  const bool all = rank_count == pl->c;
  const std::vector<WorkItem>* l_all;
  const std::vector<WorkItem>* l_rank;
  const std::vector<int32_t>* off;
  size_t o_all, o_rank;
  if (k == kPairRows) {
    l_all = &pl->quads_all; l_rank = &pl->quads_rank; off = &pl->quad_rank_off;
    o_all = pl->ws.quads_all; o_rank = pl->ws.quads_rank;
  } else if (pair_heads) {
    l_all = &pl->tiles_all; l_rank = &pl->tiles_rank; off = &pl->tile_rank_off;
    o_all = pl->ws.tiles_all; o_rank = pl->ws.tiles_rank;
  } else {
    l_all = &pl->pairs_all; l_rank = &pl->pairs_rank; off = &pl->pair_rank_off;
    o_all = pl->ws.pairs_all; o_rank = pl->ws.pairs_rank;
  }
  ItemRange r;
  r.list = all ? l_all : l_rank;
  r.ws_off = all ? o_all : o_rank;
  r.first = all ? 0 : size_t((*off)[rank_begin]);
  r.n = all ? l_all->size() : size_t((*off)[rank_begin + rank_count] - (*off)[rank_begin]);
  return r;
}

// CTAs of a launch over n work items.
int64_t grid_for(KernelChoice k, bool pair_heads, int64_t n, int h_q) {
  if (k == kPairRows) return n * h_q * 2;
  return n * (pair_heads ? h_q / 2 : h_q);
}

std::mutex g_pair_attr_mu;
bool g_pair_attr_done[256] = {};

zz_status_t ensure_pair_attr() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= 256) return fail(ZZ_ERR_UNSUPPORTED, "device ordinal above 255");
  std::lock_guard<std::mutex> lock(g_pair_attr_mu);
  if (!g_pair_attr_done[dev]) {
    e = cudaFuncSetAttribute(attn_fwd_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg::kSmem);
    if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("cudaFuncSetAttribute: ") + cudaGetErrorString(e));
    g_pair_attr_done[dev] = true;
  }
  return ZZ_OK;
}

// Tensor maps of the pair kernel (K boxes of at most 64 rows: a CTA loads 64
// keys of each K tile) and its one-time attribute; enqueues nothing.
zz_status_t prepare_pair(const void* q, int64_t q_rows, const void* k_pool, const void* v_pool,
                         int64_t num_slots, int h_q, int h_kv, int page_size, CUtensorMap* tq,
                         CUtensorMap* tk, CUtensorMap* tv, Params& p) {
  if (zz_status_t e = get_encoder()) return e;
  const int vbox = page_size >= 128 ? 128 : page_size;
  const int kbox = vbox < 64 ? vbox : 64;
  if (zz_status_t e = encode_3d(tq, q, 128, h_q, q_rows, 128)) return e;
  if (zz_status_t e = encode_3d(tk, k_pool, 128, h_kv, num_slots, kbox)) return e;
  if (zz_status_t e = encode_3d(tv, v_pool, 128, h_kv, num_slots, vbox)) return e;
  if (zz_status_t e = ensure_pair_attr()) return e;
  p.box_rows = vbox;
  // Items per scheduling chunk: one K/V head's CTAs of a chunk fill every SM
  // once (rows mode: 2 x group CTAs per K/V head and item).
  p.chunk_items = p.pair_rows ? std::max(1, (device_sm_count() + 2 * p.group - 1) / (2 * p.group))
                              : chunk_items_for(p.groups_per_kv);
  return ZZ_OK;
}

// Clusters of two CTAs along x (grid from grid_for).
zz_status_t enqueue_pair(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, int64_t grid,
                         const Params& p, cudaStream_t stream) {
  attn_fwd_pair<<<unsigned(grid), kThreads, PairCfg::kSmem, stream>>>(tq, tk, tv, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("attn_fwd_pair launch: ") + cudaGetErrorString(e));
  return ZZ_OK;
}

template <int D>
zz_status_t launch_bf16(const zz_plan_t* pl, int rank_begin, int rank_count, const void* q,
                        const void* k_pool, const void* v_pool, int64_t num_slots,
                        const int32_t* page_table, int max_pages, int page_size, void* out,
                        float* lse, int h_q, int h_kv, float scale, int causal, cudaStream_t stream) {
  using C = Cfg<D>;
  const int box_rows = page_size >= 128 ? 128 : page_size;
  const int64_t q_rows = int64_t(rank_count) * pl->M;
  const char* ws = static_cast<const char*>(pl->dev_ws);
  Params p{};
  p.halves = reinterpret_cast<const HalfDesc*>(ws + pl->ws.halves);
  p.page_table = page_table;
  p.k_pool = static_cast<const __nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<const __nv_bfloat16*>(v_pool);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.status = reinterpret_cast<int*>(const_cast<char*>(ws) + pl->ws.status);
  p.num_slots = num_slots;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = h_q / h_kv;
  p.pair_heads = (p.group % 2 == 0) ? 1 : 0;
  p.head_groups = p.pair_heads ? h_q / 2 : h_q;
  p.groups_per_kv = p.pair_heads ? p.group / 2 : p.group;
  p.M = pl->M;
  p.rank_begin = rank_begin;
  p.max_pages = max_pages;
  p.page_size = page_size;
  p.box_rows = box_rows;
  if (num_slots > int64_t(INT32_MAX) - page_size) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: num_slots too large");
  p.num_pages = int((num_slots + page_size - 1) / page_size);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = 1000000000ull;   // 1 s per wait
  p.causal = causal;
  const KernelChoice kc = kernel_for(D, p.group);
  p.pair_rows = kc == kPairRows ? 1 : 0;
  const ItemRange ir = items_for(pl, kc, p.pair_heads != 0, rank_begin, rank_count);
  p.items = reinterpret_cast<const WorkItem*>(ws + ir.ws_off) + ir.first;
  const int64_t grid = grid_for(kc, p.pair_heads != 0, int64_t(ir.n), h_q);
  if (grid == 0) return ZZ_OK;
  if (grid > INT32_MAX) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: grid too large");
  p.n_items = int(ir.n);
  if (kc != kSingleCta) {
    CUtensorMap pq, pk, pv;
    if (zz_status_t e = prepare_pair(q, q_rows, k_pool, v_pool, num_slots, h_q, h_kv, page_size, &pq, &pk, &pv, p))
      return e;
    return enqueue_pair(pq, pk, pv, grid, p, stream);
  }
  if constexpr (D == 128) {
    return fail(ZZ_ERR_UNSUPPORTED, "head_dim 128 runs on the CTA-pair kernel only");   // kernel_for never gets here
  } else {
    if (zz_status_t e = get_encoder()) return e;
    CUtensorMap tq, tk, tv;
    if (zz_status_t e = encode_3d(&tq, q, D, h_q, q_rows, 128)) return e;
    if (zz_status_t e = encode_3d(&tk, k_pool, D, h_kv, num_slots, box_rows)) return e;
    if (zz_status_t e = encode_3d(&tv, v_pool, D, h_kv, num_slots, box_rows)) return e;
    p.chunk_items = chunk_items_for(p.groups_per_kv);
    if (zz_status_t e = ensure_smem_attr<D>()) return e;
    attn_fwd_sm100<D><<<unsigned(grid), kThreads, C::kSmem, stream>>>(tq, tk, tv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("attn_fwd_sm100 launch: ") + cudaGetErrorString(e));
    return ZZ_OK;
  }
}

bool aligned16(const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15u) == 0; }


// ---------------------------------------------------------------- allocation-free variant
// Scratch of zz_attn_prefill_noalloc: the half table, the work list and the
// status word live here instead of in a caller-allocated workspace.  Every GPU
// that loads the library keeps this array until the process exits.
// Layout: [status word (16 B) | pad to 256 | half table | pad to 256 | work items].
constexpr size_t kStaticScratchBytes = size_t(1) << 20;   // 1 MiB
constexpr size_t kStaticHalvesOff = 256;
__device__ __align__(256) static unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};   // device address of g_static_scratch, per device ordinal

// The tables reach the static array as kernel parameters: the runtime copies a
// launch's parameters into its command stream when the launch is enqueued, so
// this needs neither a staging buffer (no host or device allocation) nor a
// copy from pageable memory (which would wait for the stream).  One launch
// carries up to kFillBytes; the first one also clears the status word.
constexpr int kFillWords = 2040;
constexpr uint32_t kFillBytes = kFillWords * 16;
struct FillArgs {
  uint32_t offset;        // destination byte offset in g_static_scratch (16-byte aligned)
  uint32_t nbytes;        // bytes of data[] to store (a multiple of 16)
  uint32_t clear_status;  // 1: also zero the 16-byte status word
  uint32_t pad;
  uint4 data[kFillWords];
};
static_assert(sizeof(FillArgs) <= 32764, "kernel parameters are limited to 32764 bytes");

__global__ void __launch_bounds__(256) static_scratch_fill(const __grid_constant__ FillArgs a) {
  uint4* dst = reinterpret_cast<uint4*>(g_static_scratch + a.offset);
  for (uint32_t i = threadIdx.x; i < a.nbytes / 16; i += blockDim.x) dst[i] = a.data[i];
  if (a.clear_status && threadIdx.x == 0)
    *reinterpret_cast<uint4*>(g_static_scratch) = make_uint4(0u, 0u, 0u, 0u);
}

template <int D>
zz_status_t launch_bf16_static(const zz_plan_t* pl, int rank_begin, int rank_count, const void* q,
                               const void* k_pool, const void* v_pool, int64_t num_slots,
                               const int32_t* page_table, int max_pages, int page_size, void* out,
                               float* lse, int h_q, int h_kv, float scale, cudaStream_t stream) {
  using C = Cfg<D>;
  const int group = h_q / h_kv;
  const bool pair_heads = group % 2 == 0;
  const KernelChoice kc = kernel_for(D, group);
  const ItemRange ir = items_for(pl, kc, pair_heads, rank_begin, rank_count);
  const std::vector<WorkItem>& list = *ir.list;
  const size_t first = ir.first;
  const size_t n_items = ir.n;
  const size_t halves_bytes = pl->halves.size() * sizeof(HalfDesc);
  const size_t items_off = (kStaticHalvesOff + halves_bytes + 255) & ~size_t(255);
  const size_t items_bytes = n_items * sizeof(WorkItem);
  const size_t need = items_off + items_bytes;
  // ---- every check comes before anything is enqueued ----
  if (need > kStaticScratchBytes)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: plan tables need " + std::to_string(need) +
                                        " bytes, more than the static scratch of " +
                                        std::to_string(kStaticScratchBytes) + " bytes");
  if (num_slots > int64_t(INT32_MAX) - page_size)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: num_slots too large");
  if (n_items == 0) return ZZ_OK;
  const int head_groups = pair_heads ? h_q / 2 : h_q;
  const int64_t grid = grid_for(kc, pair_heads, int64_t(n_items), h_q);
  if (grid > INT32_MAX) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: grid too large");
  if (zz_status_t e = get_encoder()) return e;
  const int box_rows = page_size >= 128 ? 128 : page_size;
  CUtensorMap tq, tk, tv;
  if (zz_status_t st = encode_3d(&tq, q, D, h_q, int64_t(rank_count) * pl->M, 128)) return st;
  if (zz_status_t st = encode_3d(&tk, k_pool, D, h_kv, num_slots, box_rows)) return st;
  if (zz_status_t st = encode_3d(&tv, v_pool, D, h_kv, num_slots, box_rows)) return st;
  const bool pair = kc != kSingleCta;
  if constexpr (D != 128) {
    if (!pair)
      if (zz_status_t e = ensure_smem_attr<D>()) return e;
  }
  void* base = nullptr;
  if (zz_status_t e = static_scratch_address(&base)) return e;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(ZZ_ERR_CUDA, "zz_attn_prefill_noalloc: cudaGetDevice");
  char* sc = static_cast<char*>(base);
  Params p{};
  p.halves = reinterpret_cast<const HalfDesc*>(sc + kStaticHalvesOff);
  p.items = reinterpret_cast<const WorkItem*>(sc + items_off);
  p.status = reinterpret_cast<int*>(sc);
  p.page_table = page_table;
  p.k_pool = static_cast<const __nv_bfloat16*>(k_pool);
  p.v_pool = static_cast<const __nv_bfloat16*>(v_pool);
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.num_slots = num_slots;
  p.h_q = h_q;
  p.h_kv = h_kv;
  p.group = group;
  p.pair_heads = pair_heads ? 1 : 0;
  p.head_groups = head_groups;
  p.groups_per_kv = pair_heads ? group / 2 : group;
  p.M = pl->M;
  p.rank_begin = rank_begin;
  p.max_pages = max_pages;
  p.page_size = page_size;
  p.box_rows = box_rows;
  p.num_pages = int((num_slots + page_size - 1) / page_size);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.timeout_ns = 1000000000ull;
  p.causal = 1;
  p.pair_rows = kc == kPairRows ? 1 : 0;
  p.n_items = int(n_items);
  p.chunk_items = chunk_items_for(p.groups_per_kv);
  if (pair)
    if (zz_status_t e = prepare_pair(q, int64_t(rank_count) * pl->M, k_pool, v_pool, num_slots, h_q, h_kv,
                                     page_size, &tq, &tk, &tv, p))
      return e;
  // ---- enqueue: the tables (in launches of up to kFillBytes), then the attention ----
  // Bytes [kStaticHalvesOff, need) of the array's image: the half table, zeros
  // up to items_off, then this call's work items.
  const char* halves_src = reinterpret_cast<const char*>(pl->halves.data());
  const char* items_src = reinterpret_cast<const char*>(list.data() + first);
  FillArgs fa;
  bool first_fill = true;
  for (size_t at = kStaticHalvesOff; at < need; at += kFillBytes) {
    const size_t len = std::min<size_t>(kFillBytes, need - at);
    const size_t padded = (len + 15) & ~size_t(15);
    char* dst = reinterpret_cast<char*>(fa.data);
    std::memset(dst, 0, padded);
    const size_t h_lo = std::max(at, kStaticHalvesOff), h_hi = std::min(at + len, kStaticHalvesOff + halves_bytes);
    if (h_lo < h_hi) std::memcpy(dst + (h_lo - at), halves_src + (h_lo - kStaticHalvesOff), h_hi - h_lo);
    const size_t i_lo = std::max(at, items_off), i_hi = std::min(at + len, need);
    if (i_lo < i_hi) std::memcpy(dst + (i_lo - at), items_src + (i_lo - items_off), i_hi - i_lo);
    fa.offset = uint32_t(at);
    fa.nbytes = uint32_t(padded);
    fa.clear_status = first_fill ? 1u : 0u;
    fa.pad = 0;
    static_scratch_fill<<<1, 256, 0, stream>>>(fa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("static_scratch_fill launch: ") + cudaGetErrorString(e));
    first_fill = false;
  }
  pl->noalloc_dev.store(dev);
  if (pair) return enqueue_pair(tq, tk, tv, grid, p, stream);
  if constexpr (D == 128) {
    return fail(ZZ_ERR_UNSUPPORTED, "head_dim 128 runs on the CTA-pair kernel only");   // kernel_for never gets here
  } else {
    attn_fwd_sm100<D><<<unsigned(grid), kThreads, C::kSmem, stream>>>(tq, tk, tv, p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("attn_fwd_sm100 launch: ") + cudaGetErrorString(e));
    return ZZ_OK;
  }
}

}  // namespace

// Device address of the static scratch on the current device.  In host code the
// array's name is only a stand-in; the address must come from the runtime,
// looked up once per device with that device current.
zz_status_t static_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(ZZ_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(ZZ_ERR_UNSUPPORTED, "device ordinal above 255");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_static_scratch);
    if (e != cudaSuccess || !ptr)
      return fail(ZZ_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return ZZ_OK;
}

std::mutex g_sm_mu;
int g_sm_count[256] = {};

int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 148;
  std::lock_guard<std::mutex> lock(g_sm_mu);
  if (!g_sm_count[dev]) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    g_sm_count[dev] = sms;
  }
  return g_sm_count[dev];
}
}  // namespace zz

extern "C" zz_status_t zz_attn_prefill_ex(const zz_plan_t* plan, int rank_begin, int rank_count,
                                          const void* q, const void* k_pool, const void* v_pool,
                                          int64_t num_slots, const int32_t* page_table, int max_pages,
                                          int page_size, void* out, float* lse, int h_q, int h_kv,
                                          int d, float softmax_scale, zz_dtype_t dtype, uint32_t flags,
                                          void* stream) {
  ZZ_NVTX("zz_attn_prefill_ex");
  using namespace zz;
  if (flags & ~uint32_t(ZZ_ATTN_NONCAUSAL)) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: unknown flags");
  const int causal = (flags & ZZ_ATTN_NONCAUSAL) ? 0 : 1;
  if (!plan || !q || !k_pool || !v_pool || !page_table || !out)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: NULL argument");
  if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: num_heads (" + std::to_string(h_q) +
                                        ") must be a multiple of num_kv_heads (" + std::to_string(h_kv) + ")");
  if (!plan->dev_ws) return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: plan not uploaded");
  if (rank_count <= 0 || rank_begin < 0 || rank_begin + rank_count > plan->c)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: rank range outside [0, cp_size)");
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: pointers must be 16-byte aligned");
  if (page_size <= 0 || max_pages <= 0 || num_slots <= 0)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: page_size, max_pages and num_slots must be positive");
  for (int s = 0; s < plan->bs; ++s) {
    int32_t kv_max = 0;
    for (int r = 0; r < plan->c; ++r) kv_max = std::max(kv_max, plan->kv_next[r][s]);
    if ((int64_t(kv_max) + page_size - 1) / page_size > max_pages)
      return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill: page_table rows shorter than the kv lengths need");
  }
  if (d != 64 && d != 128) return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill: head_dim must be 64 or 128");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  auto s = static_cast<cudaStream_t>(stream);
  if (dtype == ZZ_FP32)
    return launch_attn_simt_fp32(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                                 max_pages, page_size, out, lse, h_q, h_kv, d, scale, causal, s);
  if (dtype != ZZ_BF16) return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill: dtype must be bf16 or fp32");
  const bool ps_ok = page_size == 8 || page_size == 16 || page_size == 32 || page_size == 64 ||
                     page_size % 128 == 0;
  if (!ps_ok)
    return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill: bf16 page_size must be 8, 16, 32, 64 or a multiple of 128");
  if (d == 128)
    return launch_bf16<128>(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                            max_pages, page_size, out, lse, h_q, h_kv, scale, causal, s);
  return launch_bf16<64>(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                         max_pages, page_size, out, lse, h_q, h_kv, scale, causal, s);
}

extern "C" zz_status_t zz_attn_prefill(const zz_plan_t* plan, int rank_begin, int rank_count,
                                       const void* q, const void* k_pool, const void* v_pool,
                                       int64_t num_slots, const int32_t* page_table, int max_pages,
                                       int page_size, void* out, float* lse, int h_q, int h_kv, int d,
                                       float softmax_scale, zz_dtype_t dtype, void* stream) {
  return zz_attn_prefill_ex(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                            max_pages, page_size, out, lse, h_q, h_kv, d, softmax_scale, dtype, 0u, stream);
}

// Allocation-free variant of zz_attn_prefill (bf16): same arguments, but the
// plan's device tables go into the library's static scratch array instead of
// the workspace given to zz_plan_upload (which need not have been called).
extern "C" zz_status_t zz_attn_prefill_noalloc(const zz_plan_t* plan, int rank_begin, int rank_count,
                                               const void* q, const void* k_pool, const void* v_pool,
                                               int64_t num_slots, const int32_t* page_table,
                                               int max_pages, int page_size, void* out, float* lse,
                                               int h_q, int h_kv, int d, float softmax_scale,
                                               zz_dtype_t dtype, void* stream) {
  ZZ_NVTX("zz_attn_prefill_noalloc");
  using namespace zz;
  if (!plan || !q || !k_pool || !v_pool || !page_table || !out)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: NULL argument");
  if (h_q <= 0 || h_kv <= 0 || h_q % h_kv != 0)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: num_heads (" + std::to_string(h_q) +
                                        ") must be a multiple of num_kv_heads (" + std::to_string(h_kv) + ")");
  if (rank_count <= 0 || rank_begin < 0 || rank_begin + rank_count > plan->c)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: rank range outside [0, cp_size)");
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) || !aligned16(out) ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u) || (reinterpret_cast<uintptr_t>(lse) & 3u))
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: pointers must be 16-byte aligned");
  if (page_size <= 0 || max_pages <= 0 || num_slots <= 0)
    return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: page_size, max_pages and num_slots must be positive");
  for (int s = 0; s < plan->bs; ++s) {
    int32_t kv_max = 0;
    for (int r = 0; r < plan->c; ++r) kv_max = std::max(kv_max, plan->kv_next[r][s]);
    if ((int64_t(kv_max) + page_size - 1) / page_size > max_pages)
      return fail(ZZ_ERR_INVALID_ARG, "zz_attn_prefill_noalloc: page_table rows shorter than the kv lengths need");
  }
  if (dtype != ZZ_BF16) return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill_noalloc: dtype must be bf16");
  if (d != 64 && d != 128) return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill_noalloc: head_dim must be 64 or 128");
  const bool ps_ok = page_size == 8 || page_size == 16 || page_size == 32 || page_size == 64 ||
                     page_size % 128 == 0;
  if (!ps_ok)
    return fail(ZZ_ERR_UNSUPPORTED, "zz_attn_prefill_noalloc: page_size must be 8, 16, 32, 64 or a multiple of 128");
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(float(d));
  auto s = static_cast<cudaStream_t>(stream);
  if (d == 128)
    return launch_bf16_static<128>(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                                   max_pages, page_size, out, lse, h_q, h_kv, scale, s);
  return launch_bf16_static<64>(plan, rank_begin, rank_count, q, k_pool, v_pool, num_slots, page_table,
                                max_pages, page_size, out, lse, h_q, h_kv, scale, s);
}
