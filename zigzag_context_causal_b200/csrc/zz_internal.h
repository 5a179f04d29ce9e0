// Internal declarations shared by the host planner and the CUDA entry points.
#pragma once

#include <atomic>
#include <cstdint>
#include <string>
#include <vector>

#include "../../include/zz.h"

namespace zz {

// Query rows per work tile; the work lists are built for this tile height.
constexpr int kTileM = 128;
// Keys per K/V tile of the attention kernels (used for longest-first costs).
constexpr int kTileN = 128;

// One zigzag half of one sequence on one rank (device table entry, 32 bytes).
struct HalfDesc {
  int32_t rank;       // virtual rank r
  int32_t row0;       // first rank-local row of this half in the [M] layout
  int32_t lq;         // query rows (block size)
  int32_t kv_len;     // keys visible to the half (prefix + blocks 0..own)
  int32_t seq;        // sequence index (page-table row)
  int32_t kv_pos0;    // position of query row 0 = kv_len - lq
  int32_t half;       // 0 = prev, 1 = next
  int32_t kv_full;    // prefix + whole extend length: the keys a non-causal half sees
};

// One unit of attention work: rows [tile*128, tile*128+128) of a half, or for
// pair lists the two tiles 2*tile and 2*tile+1, or for quad lists the four
// tiles 4*tile .. 4*tile+3.
struct WorkItem {
  int32_t half_id;
  int32_t tile;
};

// Bits of the device status word (kernels OR them in; zz_plan_device_status reads them).
constexpr int kStatusTimeout = 1;   // a bounded wait gave up
constexpr int kStatusBadPage = 4;   // a page_table entry pointed outside the pool

struct Workspace {  // byte offsets into the device workspace
  size_t src_row, rank_tok, halves, tiles_all, tiles_rank, pairs_all, pairs_rank, quads_all, quads_rank,
      status, total;
};

}  // namespace zz

struct zz_plan {
  int c = 0, bs = 0;
  int64_t T = 0;
  int M = 0;
  std::vector<int32_t> ext, prefix, split_list, cp_reverse_index, reverse_split_len;
  std::vector<int32_t> per_rank, max_rank_len;
  std::vector<std::vector<int32_t>> blocks;                       // [bs][2c]
  std::vector<std::vector<int32_t>> zigzag_index;                 // [c][2bs]
  std::vector<std::vector<int32_t>> kv_prev, kv_next, q_prev, q_next;  // [c][bs]
  std::vector<std::vector<int32_t>> cu_prev, cu_next;             // [c][bs+1]
  std::vector<int32_t> total_prev, total_next, max_q_prev, max_q_next;  // [c]
  std::vector<int32_t> src_row;                                   // [T]
  std::vector<int32_t> rank_tok;                                  // [c*M]: inverse of src_row, -1 = pad
  int64_t causal_pairs = 0;
  // device tables, host copies
  std::vector<zz::HalfDesc> halves;                               // [c*2*bs]
  std::vector<zz::WorkItem> tiles_all, tiles_rank, pairs_all, pairs_rank, quads_all, quads_rank;
  std::vector<int32_t> tile_rank_off, pair_rank_off, quad_rank_off;   // [c+1]
  zz::Workspace ws{};
  void* dev_ws = nullptr;
  void* staging = nullptr;   // pinned host image of the workspace, made at the first upload
  void* staging_dev = nullptr;   // the same image as the device sees it (mapped pinned memory)
  // Device ordinal of the last zz_attn_prefill_noalloc call made with this plan
  // (-1: none); zz_plan_device_status then also reads the static status word.
  mutable std::atomic<int> noalloc_dev{-1};
};

namespace zz {
zz_status_t fail(zz_status_t st, const std::string& msg);
zz_status_t ok();
// Device address of the allocation-free entry point's static scratch on the
// current device (its first 16 bytes are that entry point's status word).
zz_status_t static_scratch_address(void** out);
// Streaming multiprocessors of the current device (cached per device ordinal).
int device_sm_count();
}  // namespace zz
