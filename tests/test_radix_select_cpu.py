"""The selectors' radix selection, checked on the CPU.

Both selectors find "the k-th best key" of a dt row: the k-th largest
composite key (float32 bits of dt, then 0xFFFFFFFF - j, so the lower index
wins ties; page "Transformers 中的 Doge 小语言模型完全指南", section
"动态掩码注意力（DMA）：从缓存 value states 生成稀疏掩码", step 3, keeps the
keep_window_size best keys of a row).  They select by most-significant digit:
  1. bits shared by every dt value are skipped (an OR / AND pass);
  2. 11-bit digits are histogrammed from the top, keeping the bin that holds
     the k-th largest, until at most `cap` candidates remain;
  3. the candidates' composite keys are selected the same way, down into the
     index bits;
  4. if all 32 dt bits are fixed and more than `cap` candidates remain (exact
     ties, e.g. A = 0 makes every dt 1), the answer is the tied key with the
     k-th smallest index.
This test restates those steps in plain Python and checks them against a
sort, on rows with random values, few distinct values, all-equal values and
values that differ only in their low bits, with small and large candidate caps.
"""
import numpy as np

from oracle import dma_oracle as oracle


def _hi_match(x, p, hb):
    return True if hb >= 63 else (x >> (hb + 1)) == (p >> (hb + 1))


def _find_bin_from_top(hist, k):
    acc = 0
    for b in range(len(hist) - 1, -1, -1):
        if acc + hist[b] >= k:
            return b, k - acc, hist[b]
        acc += hist[b]
    raise AssertionError("k exceeds the histogram total")


def _digit_select(values, width, k, stop):
    """Most-significant-digit selection of the k-th largest of `values`
    (integers of `width` bits) until `stop(count)`; returns (prefix, hb, k, count)."""
    vor, vand = 0, (1 << width) - 1
    for x in values:
        vor |= x
        vand &= x
    vary = vor ^ vand
    hb = vary.bit_length() - 1
    prefix = vand if hb < 0 else (vand & ~((2 << hb) - 1))
    count = len(values)
    while hb >= 0 and not stop(count):
        s = hb - 10 if hb >= 10 else 0
        nb = 1 << (hb - s + 1)
        hist = [0] * nb
        for x in values:
            if _hi_match(x, prefix, hb):
                hist[(x >> s) & (nb - 1)] += 1
        b, k, count = _find_bin_from_top(hist, k)
        prefix |= b << s
        hb = s - 1
    return prefix, hb, k, count


def select_kth(dt_row, n, k, cap):
    bits = [int(b) for b in np.asarray(dt_row[:n], np.float32).view(np.uint32)]
    prefix, hb, k, count = _digit_select(bits, 32, k, lambda c: c <= cap)
    if count <= cap:
        cand = [oracle.composite_key(dt_row[j], j) for j in range(n) if _hi_match(bits[j], prefix, hb)]
        p2, hb2, _, c2 = _digit_select(cand, 64, k, lambda c: c <= 1)
        match = [c for c in cand if _hi_match(c, p2, hb2)]
        assert len(match) == 1
        return match[0]
    # every candidate has dt bits == prefix: the k-th smallest tied index
    tied = [j for j in range(n) if bits[j] == prefix]
    return oracle.composite_key(dt_row[tied[k - 1]], tied[k - 1])


def _rows(rng):
    yield rng.uniform(0.0, 1.0, 5000).astype(np.float32)
    yield rng.choice(np.array([0.125, 0.5, 0.75, 1.0], np.float32), 6000)
    yield np.ones(3000, np.float32)
    base = np.float32(0.4)
    yield (base.view(np.uint32) + rng.integers(0, 64, 4000).astype(np.uint32)).view(np.float32)
    x = rng.normal(0.0, 0.64, 8000)
    yield np.exp(-1.3 * np.log1p(np.exp(x))).astype(np.float32)


def test_radix_selection_equals_sorting():
    rng = np.random.default_rng(8)
    for row in _rows(rng):
        n_max = len(row)
        keys_desc = None
        for cap in (16, 4096):
            for _ in range(6):
                n = int(rng.integers(1, n_max + 1))
                k = int(rng.integers(1, n + 1))
                keys_desc = sorted((oracle.composite_key(row[j], j) for j in range(n)), reverse=True)
                assert select_kth(row, n, k, cap) == keys_desc[k - 1], (n, k, cap)
