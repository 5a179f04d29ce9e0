// Host planner: the zigzag metadata of every rank, and the device tables the
// kernels read.  Follows "sgl-project--sglang/python/sglang/srt/layers/cp/
// zigzag.py", ZigzagCPStrategy.can_apply and ZigzagCPStrategy.build_metadata.
// O(bs * c^2) integer work; no CUDA call is made here except in zz_plan_upload.
#include <algorithm>
#include <cstring>
#include <numeric>
#include <string>

#include <cuda_runtime.h>

#include "nvtx_range.h"
#include "zz_internal.h"

namespace {
thread_local std::string g_last_error;

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int64_t pairs_of(int64_t lq, int64_t kv_len) {
  return lq * (kv_len - lq) + lq * (lq + 1) / 2;
}
}  // namespace

namespace zz {
zz_status_t fail(zz_status_t st, const std::string& msg) {
  g_last_error = msg;
  return st;
}
zz_status_t ok() { return ZZ_OK; }
}  // namespace zz

extern "C" const char* zz_last_error(void) { return g_last_error.c_str(); }

static void build_tables(zz_plan* p) {
  using zz::HalfDesc;
  using zz::WorkItem;
  const int c = p->c, bs = p->bs, nblk = 2 * c;
  // ---- natural token -> row of the rank-ordered padded layout ----
  // Token i of sequence s lies in block j; block j is rank j's prev half
  // (j < c) or rank 2c-1-j's next half.  Its rank-local row is the half's
  // start (cu_seqlens of that half, plus total_q_prev for next halves) plus
  // the offset inside the block.
  p->src_row.assign(p->T, 0);
  int64_t t = 0;
  for (int s = 0; s < bs; ++s) {
    for (int j = 0; j < nblk; ++j) {
      const bool is_prev = j < c;
      const int r = is_prev ? j : nblk - 1 - j;
      const int32_t start = is_prev ? p->cu_prev[r][s] : p->total_prev[r] + p->cu_next[r][s];
      for (int o = 0; o < p->blocks[s][j]; ++o)
        p->src_row[t++] = int32_t(int64_t(r) * p->M + start + o);
    }
  }
  // ---- rank-ordered row -> natural token (padding rows: -1) ----
  p->rank_tok.assign(size_t(c) * p->M, -1);
  for (int64_t i = 0; i < p->T; ++i) p->rank_tok[p->src_row[i]] = int32_t(i);
  // ---- half descriptors, id = (r*2 + half)*bs + s ----
  p->halves.assign(size_t(c) * 2 * bs, HalfDesc{});
  for (int r = 0; r < c; ++r)
    for (int h = 0; h < 2; ++h)
      for (int s = 0; s < bs; ++s) {
        HalfDesc d{};
        d.rank = r;
        d.half = h;
        d.seq = s;
        d.lq = h == 0 ? p->q_prev[r][s] : p->q_next[r][s];
        d.kv_len = h == 0 ? p->kv_prev[r][s] : p->kv_next[r][s];
        d.row0 = h == 0 ? p->cu_prev[r][s] : p->total_prev[r] + p->cu_next[r][s];
        d.kv_pos0 = d.kv_len - d.lq;
        d.kv_full = p->prefix[s] + p->ext[s];
        p->halves[(size_t(r) * 2 + h) * bs + s] = d;
      }
  // ---- longest-first work lists ----
  struct Costed { WorkItem w; int32_t rank; int64_t cost; };
  auto kv_tiles_upto_row = [&](const HalfDesc& d, int64_t last_row) -> int64_t {
    const int64_t last_key = int64_t(d.kv_pos0) + last_row;  // inclusive
    return last_key / zz::kTileN + 1;
  };
  std::vector<Costed> tiles, pairs, quads;
  for (size_t id = 0; id < p->halves.size(); ++id) {
    const HalfDesc& d = p->halves[id];
    const int nt = (d.lq + zz::kTileM - 1) / zz::kTileM;
    for (int k = 0; k < nt; ++k) {
      const int64_t last = std::min<int64_t>(int64_t(k + 1) * zz::kTileM, d.lq) - 1;
      tiles.push_back({{int32_t(id), k}, d.rank, kv_tiles_upto_row(d, last)});
    }
    for (int k = 0; 2 * k < nt; ++k) {
      const int64_t last = std::min<int64_t>(int64_t(2 * k + 2) * zz::kTileM, d.lq) - 1;
      const int64_t first_last = std::min<int64_t>(int64_t(2 * k + 1) * zz::kTileM, d.lq) - 1;
      const int64_t cost = kv_tiles_upto_row(d, last) +
                           (2 * k + 1 < nt ? kv_tiles_upto_row(d, first_last) : 0);
      pairs.push_back({{int32_t(id), k}, d.rank, cost});
    }
    // Quads (CTA pairs, two row tiles per CTA): every tile of the quad runs to
    // the keys of its last valid row tile.
    for (int k = 0; 4 * k < nt; ++k) {
      const int64_t last = std::min<int64_t>(int64_t(4 * k + 4) * zz::kTileM, d.lq) - 1;
      quads.push_back({{int32_t(id), k}, d.rank, 4 * kv_tiles_upto_row(d, last)});
    }
  }
  auto by_cost = [](const Costed& a, const Costed& b) { return a.cost > b.cost; };
  auto by_rank_cost = [](const Costed& a, const Costed& b) {
    return a.rank != b.rank ? a.rank < b.rank : a.cost > b.cost;
  };
  auto emit = [&](std::vector<Costed> v, bool rank_major, std::vector<WorkItem>& out,
                  std::vector<int32_t>* off) {
    if (rank_major) std::stable_sort(v.begin(), v.end(), by_rank_cost);
    else std::stable_sort(v.begin(), v.end(), by_cost);
    out.clear();
    for (auto& x : v) out.push_back(x.w);
    if (off) {
      off->assign(c + 1, 0);
      for (auto& x : v) (*off)[x.rank + 1]++;
      for (int r = 0; r < c; ++r) (*off)[r + 1] += (*off)[r];
    }
  };
  emit(tiles, false, p->tiles_all, nullptr);
  emit(tiles, true, p->tiles_rank, &p->tile_rank_off);
  emit(pairs, false, p->pairs_all, nullptr);
  emit(pairs, true, p->pairs_rank, &p->pair_rank_off);
  emit(quads, false, p->quads_all, nullptr);
  emit(quads, true, p->quads_rank, &p->quad_rank_off);
  // ---- workspace layout ----
  zz::Workspace& w = p->ws;
  size_t at = 0;
  w.src_row = at;    at = align256(at + sizeof(int32_t) * size_t(p->T));
  w.rank_tok = at;   at = align256(at + sizeof(int32_t) * p->rank_tok.size());
  w.halves = at;     at = align256(at + sizeof(HalfDesc) * p->halves.size());
  w.tiles_all = at;  at = align256(at + sizeof(WorkItem) * p->tiles_all.size());
  w.tiles_rank = at; at = align256(at + sizeof(WorkItem) * p->tiles_rank.size());
  w.pairs_all = at;  at = align256(at + sizeof(WorkItem) * p->pairs_all.size());
  w.pairs_rank = at; at = align256(at + sizeof(WorkItem) * p->pairs_rank.size());
  w.quads_all = at;  at = align256(at + sizeof(WorkItem) * p->quads_all.size());
  w.quads_rank = at; at = align256(at + sizeof(WorkItem) * p->quads_rank.size());
  w.status = at;     at = align256(at + 4 * sizeof(int32_t));
  w.total = at;
}

extern "C" zz_status_t zz_plan_create(int cp_size, int bs, const int32_t* extend_lens,
                                      const int32_t* seq_lens, int64_t num_tokens,
                                      zz_plan_t** out) {
  if (!out) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: out is NULL");
  *out = nullptr;
  if (bs <= 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: bs must be positive");
  if (num_tokens < 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: num_tokens < 0");
  // Default extend lengths as on the page: seq_lens, else one sequence of num_tokens.
  std::vector<int64_t> ext(bs);
  if (extend_lens) {
    for (int i = 0; i < bs; ++i) ext[i] = extend_lens[i];
  } else if (seq_lens) {
    for (int i = 0; i < bs; ++i) ext[i] = seq_lens[i];
  } else {
    if (bs != 1)
      return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: bs must be 1 without length lists");
    ext[0] = num_tokens;
  }
  for (int i = 0; i < bs; ++i)
    if (ext[i] < 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: negative extend length");
  if (seq_lens)
    for (int i = 0; i < bs; ++i)
      if (seq_lens[i] < 0) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: negative seq length");
  const int64_t sum_ext = std::accumulate(ext.begin(), ext.end(), int64_t(0));
  // can_apply (checked on the lengths as given, before the pad fold-in).
  const int64_t nblk = 2 * int64_t(cp_size);
  if (cp_size <= 1)
    return zz::fail(ZZ_ERR_NOT_APPLICABLE, "zigzag CP needs cp_size > 1");
  if (num_tokens < nblk)
    return zz::fail(ZZ_ERR_NOT_APPLICABLE, "zigzag CP needs num_tokens >= 2*cp_size");
  for (int i = 0; i < bs; ++i)
    if (ext[i] < nblk)
      return zz::fail(ZZ_ERR_NOT_APPLICABLE,
                      "zigzag CP needs every extend length >= 2*cp_size (sequence " +
                          std::to_string(i) + " has " + std::to_string(ext[i]) + ")");
  if (num_tokens < sum_ext)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: num_tokens < sum(extend_lens)");
  if (num_tokens > INT32_MAX / 2)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: too many tokens for int32 rows");

  auto* p = new zz_plan();
  p->c = cp_size;
  p->bs = bs;
  // Pad fold-in.
  std::vector<int64_t> seqs;
  if (seq_lens) seqs.assign(seq_lens, seq_lens + bs);
  const int64_t pad = num_tokens - sum_ext;
  if (pad > 0) {
    ext[bs - 1] += pad;
    if (!seqs.empty()) seqs[bs - 1] += pad;
  }
  p->ext.resize(bs);
  p->prefix.assign(bs, 0);
  for (int i = 0; i < bs; ++i) {
    p->ext[i] = int32_t(ext[i]);
    if (!seqs.empty()) p->prefix[i] = int32_t(std::max<int64_t>(seqs[i] - ext[i], 0));
  }
  p->T = num_tokens;
  // Block sizes: base = L / 2c, the first L % 2c blocks get one more.
  p->blocks.assign(bs, std::vector<int32_t>(nblk));
  for (int s = 0; s < bs; ++s) {
    const int64_t base = ext[s] / nblk, rem = ext[s] % nblk;
    for (int j = 0; j < nblk; ++j) {
      p->blocks[s][j] = int32_t(base + (j < rem ? 1 : 0));
      p->split_list.push_back(p->blocks[s][j]);
    }
  }
  const int c = cp_size;
  p->per_rank.assign(c, 0);
  for (int r = 0; r < c; ++r)
    for (int s = 0; s < bs; ++s) p->per_rank[r] += p->blocks[s][r] + p->blocks[s][nblk - 1 - r];
  p->M = *std::max_element(p->per_rank.begin(), p->per_rank.end());
  if (int64_t(p->M) * c > INT32_MAX) {
    delete p;
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: c*M exceeds int32 rows");
  }
  p->max_rank_len.assign(c, p->M);
  p->zigzag_index.assign(c, {});
  for (int r = 0; r < c; ++r) {
    for (int s = 0; s < bs; ++s) p->zigzag_index[r].push_back(int32_t(s * nblk + r));
    for (int s = 0; s < bs; ++s) p->zigzag_index[r].push_back(int32_t(s * nblk + nblk - 1 - r));
  }
  // Gathered chunk q = r*2bs + s is rank r's prev block of seq s, and
  // r*2bs + bs + s its next block.  Natural order of seq s: blocks 0..c-1 are
  // ranks 0..c-1's prev chunks, blocks c..2c-1 are ranks c-1..0's next chunks.
  for (int s = 0; s < bs; ++s) {
    for (int j = 0; j < nblk; ++j) {
      const int r = j < c ? j : int(nblk) - 1 - j;
      p->cp_reverse_index.push_back(int32_t(r * 2 * bs + (j < c ? 0 : bs) + s));
    }
  }
  for (int r = 0; r < c; ++r) {
    for (int s = 0; s < bs; ++s) p->reverse_split_len.push_back(p->blocks[s][r]);
    for (int s = 0; s < bs; ++s) p->reverse_split_len.push_back(p->blocks[s][nblk - 1 - r]);
  }
  p->kv_prev.assign(c, std::vector<int32_t>(bs));
  p->kv_next = p->q_prev = p->q_next = p->kv_prev;
  p->cu_prev.assign(c, std::vector<int32_t>(bs + 1, 0));
  p->cu_next = p->cu_prev;
  p->total_prev.assign(c, 0);
  p->total_next.assign(c, 0);
  p->max_q_prev.assign(c, 0);
  p->max_q_next.assign(c, 0);
  for (int r = 0; r < c; ++r) {
    for (int s = 0; s < bs; ++s) {
      int64_t upto_prev = 0, upto_next = 0;
      for (int j = 0; j <= r; ++j) upto_prev += p->blocks[s][j];
      for (int j = 0; j < nblk - r; ++j) upto_next += p->blocks[s][j];
      p->kv_prev[r][s] = int32_t(p->prefix[s] + upto_prev);
      p->kv_next[r][s] = int32_t(p->prefix[s] + upto_next);
      p->q_prev[r][s] = p->blocks[s][r];
      p->q_next[r][s] = p->blocks[s][nblk - 1 - r];
      p->cu_prev[r][s + 1] = p->cu_prev[r][s] + p->q_prev[r][s];
      p->cu_next[r][s + 1] = p->cu_next[r][s] + p->q_next[r][s];
      p->max_q_prev[r] = std::max(p->max_q_prev[r], p->q_prev[r][s]);
      p->max_q_next[r] = std::max(p->max_q_next[r], p->q_next[r][s]);
      p->causal_pairs += pairs_of(p->q_prev[r][s], p->kv_prev[r][s]) +
                         pairs_of(p->q_next[r][s], p->kv_next[r][s]);
    }
    p->total_prev[r] = p->cu_prev[r][bs];
    p->total_next[r] = p->cu_next[r][bs];
  }
  // The page's own asserts.
  {
    int64_t ssum = 0;
    for (int32_t x : p->split_list) ssum += x;
    std::vector<int32_t> sorted = p->cp_reverse_index;
    std::sort(sorted.begin(), sorted.end());
    bool perm = true;
    for (size_t i = 0; i < sorted.size(); ++i) perm &= sorted[i] == int32_t(i);
    int64_t rsum = 0;
    for (int32_t x : p->per_rank) rsum += x;
    if (int64_t(p->split_list.size()) != bs * nblk || ssum != p->T || !perm || rsum != p->T) {
      delete p;
      return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_create: internal invariant violated");
    }
  }
  build_tables(p);
  *out = p;
  return ZZ_OK;
}

extern "C" void zz_plan_destroy(zz_plan_t* plan) {
  if (plan && plan->staging) cudaFreeHost(plan->staging);
  delete plan;
}

extern "C" zz_status_t zz_plan_info(const zz_plan_t* p, int rank, zz_plan_info_t* out) {
  if (!p || !out) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_info: NULL argument");
  if (rank < 0 || rank >= p->c) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_info: rank out of range");
  out->cp_size = p->c;
  out->bs = p->bs;
  out->total_tokens = p->T;
  out->max_rank_len = p->M;
  out->total_q_prev = p->total_prev[rank];
  out->total_q_next = p->total_next[rank];
  out->max_seqlen_q_prev = p->max_q_prev[rank];
  out->max_seqlen_q_next = p->max_q_next[rank];
  out->causal_pairs = p->causal_pairs;
  return ZZ_OK;
}

extern "C" zz_status_t zz_plan_get(const zz_plan_t* p, int rank, zz_field_t field, int32_t* dst,
                                   int64_t capacity, int64_t* count) {
  if (!p || !count) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_get: NULL argument");
  const bool per_rank = field == ZZ_FIELD_ZIGZAG_INDEX || field == ZZ_FIELD_KV_LEN_PREV ||
                        field == ZZ_FIELD_KV_LEN_NEXT || field == ZZ_FIELD_Q_LEN_PREV ||
                        field == ZZ_FIELD_Q_LEN_NEXT || field == ZZ_FIELD_CU_SEQLENS_Q_PREV ||
                        field == ZZ_FIELD_CU_SEQLENS_Q_NEXT;
  if (per_rank && (rank < 0 || rank >= p->c))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_get: rank out of range");
  const std::vector<int32_t>* v = nullptr;
  switch (field) {
    case ZZ_FIELD_EXTEND_LENS: v = &p->ext; break;
    case ZZ_FIELD_PREFIX: v = &p->prefix; break;
    case ZZ_FIELD_SPLIT_LIST: v = &p->split_list; break;
    case ZZ_FIELD_ZIGZAG_INDEX: v = &p->zigzag_index[rank]; break;
    case ZZ_FIELD_CP_REVERSE_INDEX: v = &p->cp_reverse_index; break;
    case ZZ_FIELD_REVERSE_SPLIT_LEN: v = &p->reverse_split_len; break;
    case ZZ_FIELD_PER_RANK_TOKENS: v = &p->per_rank; break;
    case ZZ_FIELD_MAX_RANK_LEN: v = &p->max_rank_len; break;
    case ZZ_FIELD_KV_LEN_PREV: v = &p->kv_prev[rank]; break;
    case ZZ_FIELD_KV_LEN_NEXT: v = &p->kv_next[rank]; break;
    case ZZ_FIELD_Q_LEN_PREV: v = &p->q_prev[rank]; break;
    case ZZ_FIELD_Q_LEN_NEXT: v = &p->q_next[rank]; break;
    case ZZ_FIELD_CU_SEQLENS_Q_PREV: v = &p->cu_prev[rank]; break;
    case ZZ_FIELD_CU_SEQLENS_Q_NEXT: v = &p->cu_next[rank]; break;
    case ZZ_FIELD_SRC_ROW: v = &p->src_row; break;
    case ZZ_FIELD_RANK_TOK: v = &p->rank_tok; break;
    default: return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_get: unknown field");
  }
  *count = int64_t(v->size());
  if (!dst) return ZZ_OK;
  if (capacity < int64_t(v->size()))
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_get: destination too small");
  std::memcpy(dst, v->data(), v->size() * sizeof(int32_t));
  return ZZ_OK;
}

extern "C" size_t zz_plan_workspace_bytes(const zz_plan_t* p) { return p ? p->ws.total : 0; }

namespace {
// The upload itself: plain 16-byte loads from the pinned (device-mapped) host
// image, one kernel on the caller's stream.  A copy-engine transfer
// (cudaMemcpyAsync) would queue behind other streams' host<->device copies,
// e.g. the next batch's inputs, and stall the stream for as long as they take.
__global__ void __launch_bounds__(256) upload_tables(const int4* __restrict__ src, int4* __restrict__ dst,
                                                     size_t n16) {
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += size_t(gridDim.x) * blockDim.x)
    dst[i] = src[i];
}
}  // namespace

extern "C" zz_status_t zz_plan_upload(zz_plan_t* p, void* dev, size_t bytes, void* stream) {
  ZZ_NVTX("zz_plan_upload");
  if (!p || !dev) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_upload: NULL argument");
  if (bytes < p->ws.total) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_upload: workspace too small");
  if (reinterpret_cast<uintptr_t>(dev) % 256)
    return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_upload: workspace must be 256-byte aligned");
  auto s = static_cast<cudaStream_t>(stream);
  // The tables never change after zz_plan_create: lay them out once in pinned
  // host memory exactly as in the workspace (status word zero), so that every
  // upload is one kernel that reads that image over the bus: it neither blocks
  // the calling thread nor waits for other streams' copies.
  if (!p->staging) {
    void* h = nullptr;
    cudaError_t e = cudaMallocHost(&h, p->ws.total);
    if (e != cudaSuccess)
      return zz::fail(ZZ_ERR_CUDA, std::string("zz_plan_upload: pinned staging: ") + cudaGetErrorString(e));
    char* img = static_cast<char*>(h);
    std::memset(img, 0, p->ws.total);
    struct Part { size_t off; const void* src; size_t n; } parts[] = {
        {p->ws.src_row, p->src_row.data(), p->src_row.size() * sizeof(int32_t)},
        {p->ws.rank_tok, p->rank_tok.data(), p->rank_tok.size() * sizeof(int32_t)},
        {p->ws.halves, p->halves.data(), p->halves.size() * sizeof(zz::HalfDesc)},
        {p->ws.tiles_all, p->tiles_all.data(), p->tiles_all.size() * sizeof(zz::WorkItem)},
        {p->ws.tiles_rank, p->tiles_rank.data(), p->tiles_rank.size() * sizeof(zz::WorkItem)},
        {p->ws.pairs_all, p->pairs_all.data(), p->pairs_all.size() * sizeof(zz::WorkItem)},
        {p->ws.pairs_rank, p->pairs_rank.data(), p->pairs_rank.size() * sizeof(zz::WorkItem)},
        {p->ws.quads_all, p->quads_all.data(), p->quads_all.size() * sizeof(zz::WorkItem)},
        {p->ws.quads_rank, p->quads_rank.data(), p->quads_rank.size() * sizeof(zz::WorkItem)},
    };
    for (auto& part : parts)
      if (part.n) std::memcpy(img + part.off, part.src, part.n);
    void* mapped = nullptr;
    e = cudaHostGetDevicePointer(&mapped, h, 0);
    if (e != cudaSuccess) {
      cudaFreeHost(h);
      return zz::fail(ZZ_ERR_CUDA, std::string("zz_plan_upload: mapping the staging: ") + cudaGetErrorString(e));
    }
    p->staging = h;
    p->staging_dev = mapped;
  }
  const size_t n16 = p->ws.total / 16;   // the workspace size is a multiple of 256 bytes
  const size_t blocks = std::min<size_t>((n16 + 255) / 256, 1024);
  upload_tables<<<unsigned(blocks), 256, 0, s>>>(static_cast<const int4*>(p->staging_dev), static_cast<int4*>(dev),
                                                 n16);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess)
    return zz::fail(ZZ_ERR_CUDA, std::string("zz_plan_upload: ") + cudaGetErrorString(e));
  p->dev_ws = dev;
  return ZZ_OK;
}

extern "C" zz_status_t zz_plan_device_status(const zz_plan_t* p, int32_t* flags, int clear,
                                             void* stream) {
  if (!p || !flags) return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_device_status: NULL argument");
  const int noalloc_dev = p->noalloc_dev.load();
  if (!p->dev_ws && noalloc_dev < 0)
    return zz::fail(ZZ_ERR_INVALID_ARG,
                    "zz_plan_device_status: plan neither uploaded nor used by zz_attn_prefill_noalloc");
  auto s = static_cast<cudaStream_t>(stream);
  // Status words to read: the plan's workspace word, and the static array's
  // word when this plan's last allocation-free call ran on the current device.
  char* words[2] = {nullptr, nullptr};
  int n = 0;
  if (p->dev_ws) words[n++] = static_cast<char*>(p->dev_ws) + p->ws.status;
  if (noalloc_dev >= 0) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
      return zz::fail(ZZ_ERR_CUDA, std::string("zz_plan_device_status: ") + cudaGetErrorString(e));
    if (dev == noalloc_dev) {
      void* base = nullptr;
      if (zz_status_t st = zz::static_scratch_address(&base)) return st;
      words[n++] = static_cast<char*>(base);
    } else if (!p->dev_ws) {
      return zz::fail(ZZ_ERR_INVALID_ARG, "zz_plan_device_status: make the device of the plan's last "
                                          "zz_attn_prefill_noalloc call current first");
    }
  }
  int32_t got[2] = {0, 0};
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < n && e == cudaSuccess; ++i)
    e = cudaMemcpyAsync(&got[i], words[i], sizeof(int32_t), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  for (int i = 0; i < n && e == cudaSuccess && clear; ++i)
    e = cudaMemsetAsync(words[i], 0, 4 * sizeof(int32_t), s);
  if (e != cudaSuccess)
    return zz::fail(ZZ_ERR_CUDA, std::string("zz_plan_device_status: ") + cudaGetErrorString(e));
  *flags = got[0] | got[1];
  if (*flags & zz::kStatusTimeout)
    return zz::fail(ZZ_ERR_DEVICE_TIMEOUT, "a bounded device wait gave up (pipeline stalled)");
  if (*flags & zz::kStatusBadPage)
    return zz::fail(ZZ_ERR_INVALID_ARG,
                    "a page_table entry pointed outside the pool; its keys were read as zeros");
  return ZZ_OK;
}
