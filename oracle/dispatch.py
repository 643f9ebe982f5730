"""The tuned-table lookup walk and the census deduplication rule.

Walk ([aiter#7752] "PR-specific question"; [cookbook#8] "Two amplifiers"):
the lookup probes the table at exact M; then at the next power of two when
M < 16, or at the next multiple of 16 when 16 <= M <= 256; then at the next
power of two; and gives up (a miss, which runs the per-shape default kernel;
[mi210 docs/43] section 6 "First, the good news": a miss returns None and the
default kernel runs, so partial tables cannot poison untuned shapes).
M = 6016 therefore runs the row tuned for 8192 ([cookbook#8]).

Census ([cookbook#8], review comment 1 on coverage_report.py): a server logs
one line per lookup per worker, so records are deduplicated by the key
(M, N, K, table, padded_M, library) before counting distinct hits and misses.

Parity: pinned in tests/test_oracle_dispatch.py against the worked examples
the pages print (tests/golden/padded_m_examples.txt).
"""


def next_pow2(m: int) -> int:
    p = 1
    while p < m:
        p *= 2
    return p


def probe_sequence(m: int) -> list:
    """The padded M values probed, in order, with repeats removed."""
    if m <= 0:
        raise ValueError("M must be positive")
    seq = [m]
    if m < 16:
        seq.append(next_pow2(m))
    elif m <= 256:
        seq.append(((m + 15) // 16) * 16)
    seq.append(next_pow2(m))
    out = []
    for p in seq:
        if p not in out:
            out.append(p)
    return out


def lookup(table_ms, m: int):
    """table_ms: set of padded M with a row (for one (N, K)). Returns the row's M or None (miss)."""
    for p in probe_sequence(m):
        if p in table_ms:
            return p
    return None


def census(records):
    """records: iterable of dicts with keys M, N, K, table, padded_M (None = miss), lib.

    Returns (distinct_hits, distinct_misses, drift) where drift counts distinct
    hit records whose padded_M differs from M.
    """
    seen = {}
    for r in records:
        key = (r["M"], r["N"], r["K"], r["table"], r["padded_M"], r["lib"])
        seen[key] = r
    hits = [r for r in seen.values() if r["padded_M"] is not None]
    misses = [r for r in seen.values() if r["padded_M"] is None]
    drift = sum(1 for r in hits if r["padded_M"] != r["M"])
    return len(hits), len(misses), drift
