"""Paged KV-cache gather oracle -- test infrastructure only.

Plain statement of the operation of the "PagedCacheLoadOperation" page
(Ascend Transformer Boost C API, AtbPagedCacheLoadGetWorkspaceSize members
table: keyCache / valueCache / blockTables / contextLens / key / value /
seqStarts / isSeqLensCumsumType / hasSeqStarts rows), ND cache format only.

For batch entry b with context length len_b and start s_b (seqStarts[b], or 0
without seqStarts), each logical token t < len_b lives at logical position
p = s_b + t of the sequence, i.e. in row p mod block_size of physical block
blockTables[b][p // block_size]; it is copied to packed output row o_b + t,
where o_b = len_0 + ... + len_{b-1}:

    key[o_b + t]   = keyCache[blockTables[b][p // bs], p % bs]
    value[o_b + t] = valueCache[blockTables[b][p // bs], p % bs]

contextLens holds the lengths, or, in cumulative mode, batch + 1 running
sums c with len_b = c[b+1] - c[b] (and o_b = c[b] - c[0]).  A row whose
logical block lies past the table width, or whose block id is outside
[0, num_blocks), is written as zeros and flagged.

Only tests/ and the benchmark's CPU baseline may use this module; it shares no
code with the CUDA path.  Every element is copied by an explicit loop over
batch entries and tokens -- no vectorised gather.
"""
import numpy as np


def lengths_and_offsets(context_lens, cumsum):
    """(len_b, o_b) per batch entry, from plain or cumulative context lengths."""
    c = [int(v) for v in np.asarray(context_lens).reshape(-1)]
    if cumsum:
        lens = [c[b + 1] - c[b] for b in range(len(c) - 1)]
    else:
        lens = list(c)
    offs = []
    run = 0
    for n in lens:
        offs.append(run)
        run += n
    return lens, offs, run


def paged_cache_load(key_cache, value_cache, block_tables, context_lens, seq_starts=None, cumsum=False,
                     num_tokens=None):
    """Gathers (key, value, bad_rows) from ND paged caches.

    key_cache [num_blocks, block_size, H, Dk], value_cache [num_blocks, block_size, H, Dv]
    (numpy arrays of any dtype; values are copied, never converted);
    block_tables [batch, W] int; context_lens [batch] (or [batch + 1] cumulative);
    seq_starts [batch] or None.  Returns key [T, H, Dk], value [T, H, Dv] with
    T = num_tokens (default: the total length) and the list of packed rows
    written as zeros because their block index was out of range.
    """
    key_cache = np.asarray(key_cache)
    value_cache = np.asarray(value_cache)
    tables = np.asarray(block_tables)
    lens, offs, total = lengths_and_offsets(context_lens, cumsum)
    batch = len(lens)
    num_blocks, block_size = key_cache.shape[0], key_cache.shape[1]
    width = tables.shape[1] if tables.ndim == 2 else 0
    T = total if num_tokens is None else num_tokens
    key = np.zeros((T,) + key_cache.shape[2:], dtype=key_cache.dtype)
    value = np.zeros((T,) + value_cache.shape[2:], dtype=value_cache.dtype)
    bad = []
    for b in range(batch):
        start = 0 if seq_starts is None else int(np.asarray(seq_starts).reshape(-1)[b])
        for t in range(lens[b]):
            row = offs[b] + t
            if row >= T:
                continue
            pos = start + t
            lb, within = pos // block_size, pos % block_size
            blk = int(tables[b, lb]) if 0 <= lb < width else -1
            if not (0 <= blk < num_blocks):
                bad.append(row)
                continue
            key[row] = key_cache[blk, within]
            value[row] = value_cache[blk, within]
    return key, value, bad
