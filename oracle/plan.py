"""Zigzag CP metadata, restated for all ranks at once.  TEST INFRASTRUCTURE.

Follows "sgl-project--sglang/python/sglang/srt/layers/cp/zigzag.py",
``ZigzagCPStrategy.can_apply`` and ``ZigzagCPStrategy.build_metadata``.  The
page computes the lists for one ``cp_rank``; here every rank's lists are built
so that one process can check all ``c`` virtual ranks.
"""
from __future__ import annotations

from dataclasses import dataclass, field


def can_apply(cp_size: int, num_tokens: int, extend_lens=None) -> bool:
    """zigzag.py, ``can_apply``: needs c > 1, at least 2c tokens, and every
    extend length at least 2c (the forward-mode check is a serving concern)."""
    blocks = 2 * cp_size
    if cp_size <= 1 or num_tokens < blocks:
        return False
    if extend_lens is None:
        return True
    return all(int(n) >= blocks for n in extend_lens)


def block_sizes(length: int, cp_size: int) -> list[int]:
    """zigzag.py, ``build_metadata``: a sequence is cut into 2c blocks as evenly
    as possible; the first ``length mod 2c`` blocks get one extra token."""
    nblk = 2 * cp_size
    q, r = divmod(int(length), nblk)
    return [q + 1 if j < r else q for j in range(nblk)]


@dataclass
class Plan:
    cp_size: int
    bs: int
    extend_lens: list           # after the pad fold-in
    prefix: list                # cached-prefix tokens per sequence
    blocks: list                # blocks[s][j]
    split_list: list            # concatenation of blocks, length bs*2c
    per_rank_actual_token: list  # [c]
    max_rank_len: list          # [c], all equal
    zigzag_index: list          # [c][2*bs]
    cp_reverse_index: list      # [bs*2c], rank independent
    reverse_split_len: list     # [c*2*bs]
    kv_len_prev: list           # [c][bs]
    kv_len_next: list           # [c][bs]
    q_len_prev: list            # [c][bs]  (actual_seq_q_prev)
    q_len_next: list            # [c][bs]
    cu_seqlens_q_prev: list     # [c][bs+1]
    cu_seqlens_q_next: list     # [c][bs+1]
    total_q_prev: list = field(default_factory=list)   # [c]
    total_q_next: list = field(default_factory=list)   # [c]
    max_seqlen_q_prev: list = field(default_factory=list)  # [c]
    max_seqlen_q_next: list = field(default_factory=list)  # [c]

    @property
    def total_tokens(self) -> int:
        return sum(self.extend_lens)

    @property
    def M(self) -> int:
        return self.max_rank_len[0]


def _prefix_sums(xs):
    out, acc = [0], 0
    for x in xs:
        acc += x
        out.append(acc)
    return out


def build_metadata(cp_size: int, num_tokens: int, seqs_len=None, extend_lens=None) -> Plan:
    """zigzag.py, ``build_metadata``, for every rank.

    Steps, in the page's order:
      1. default the extend lengths to ``seqs_len`` (or one sequence of
         ``num_tokens``); fold ``num_tokens - sum(extend)`` padding into the
         last sequence (and into ``seqs_len[-1]`` when both lists match);
      2. prefix offsets ``max(seqs_len - extend, 0)`` when ``seqs_len`` matches,
         else zeros;
      3. block sizes and ``split_list``;
      4. tokens per rank (block r plus block 2c-1-r of every sequence) and
         ``max_rank_len``;
      5. ``zigzag_index``: the rank's prev blocks of every sequence, then its
         next blocks;
      6. ``cp_reverse_index``: per sequence, the chunks of ranks 0..c-1 (prev)
         then ranks c-1..0 (next) of the rank-ordered gathered buffer;
      7. ``reverse_split_len``: chunk sizes of that buffer;
      8. per-sequence kv lengths (prefix plus blocks up to and including the
         rank's own block), q lengths and their exclusive prefix sums.
    """
    c = int(cp_size)
    nblk = 2 * c
    if extend_lens is None:
        extend_lens = list(seqs_len) if seqs_len else [int(num_tokens)]
    ext = [int(x) for x in extend_lens]
    pad = int(num_tokens) - sum(ext)
    seqs = None if seqs_len is None else [int(x) for x in seqs_len]
    if pad > 0:
        ext[-1] += pad
        if seqs is not None and len(seqs) == len(ext):
            seqs[-1] += pad
    bs = len(ext)
    if seqs is not None and len(seqs) == bs:
        prefix = [max(seqs[i] - ext[i], 0) for i in range(bs)]
    else:
        prefix = [0] * bs

    blocks = [block_sizes(L, c) for L in ext]
    split_list = [b for blk in blocks for b in blk]

    per_rank = [sum(blk[r] + blk[nblk - 1 - r] for blk in blocks) for r in range(c)]
    max_rank_len = [max(per_rank)] * c

    zigzag_index = []
    for r in range(c):
        prev_chunks = [s * nblk + r for s in range(bs)]
        next_chunks = [s * nblk + (nblk - 1 - r) for s in range(bs)]
        zigzag_index.append(prev_chunks + next_chunks)

    # Gathered buffer (padding trimmed) holds, for rank r, chunk numbers
    # r*2bs + s (prev block r of seq s) and r*2bs + bs + s (next block 2c-1-r).
    cp_reverse_index = []
    for s in range(bs):
        front = [r * 2 * bs + s for r in range(c)]                  # blocks 0..c-1
        back = [r * 2 * bs + bs + s for r in reversed(range(c))]    # blocks c..2c-1
        cp_reverse_index.extend(front + back)

    reverse_split_len = []
    for r in range(c):
        reverse_split_len.extend(blk[r] for blk in blocks)
        reverse_split_len.extend(blk[nblk - 1 - r] for blk in blocks)

    kv_prev, kv_next, ql_prev, ql_next = [], [], [], []
    for r in range(c):
        kv_prev.append([prefix[s] + sum(blocks[s][: r + 1]) for s in range(bs)])
        kv_next.append([prefix[s] + sum(blocks[s][: nblk - r]) for s in range(bs)])
        ql_prev.append([blocks[s][r] for s in range(bs)])
        ql_next.append([blocks[s][nblk - 1 - r] for s in range(bs)])
    cu_prev = [_prefix_sums(x) for x in ql_prev]
    cu_next = [_prefix_sums(x) for x in ql_next]

    plan = Plan(
        cp_size=c, bs=bs, extend_lens=ext, prefix=prefix, blocks=blocks,
        split_list=split_list, per_rank_actual_token=per_rank,
        max_rank_len=max_rank_len, zigzag_index=zigzag_index,
        cp_reverse_index=cp_reverse_index, reverse_split_len=reverse_split_len,
        kv_len_prev=kv_prev, kv_len_next=kv_next, q_len_prev=ql_prev,
        q_len_next=ql_next, cu_seqlens_q_prev=cu_prev, cu_seqlens_q_next=cu_next,
        total_q_prev=[x[-1] for x in cu_prev], total_q_next=[x[-1] for x in cu_next],
        max_seqlen_q_prev=[max(x) if x else 0 for x in ql_prev],
        max_seqlen_q_next=[max(x) if x else 0 for x in ql_next],
    )
    check_invariants(plan)
    return plan


def check_invariants(p: Plan) -> None:
    """zigzag.py, ``build_metadata``: the page's own asserts on the lists."""
    nblk = 2 * p.cp_size
    total = sum(p.extend_lens)
    assert len(p.split_list) == p.bs * nblk
    assert sum(p.split_list) == total
    for zi in p.zigzag_index:
        assert len(zi) == 2 * p.bs
    assert len(p.cp_reverse_index) == p.bs * nblk
    assert sorted(p.cp_reverse_index) == list(range(p.bs * nblk))
    assert sum(p.per_rank_actual_token) == total
