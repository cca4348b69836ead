"""The sorting networks of the one-thread-per-token router, checked on the CPU.

The comparators are read from the kernel source itself (the calls in sort8),
so a dropped or mistyped comparator fails here.  A comparator network sorts
every input iff it sorts every 0/1 input (Knuth, TAOCP vol. 3, 5.3.4), which
for 8 inputs is 256 cases.  The merge step (pairwise maxima of two descending
lists, one reversed, then a bitonic merge) and the k-th-largest formula used
for the threshold are checked against a plain sort on random inputs with many
ties."""
import itertools
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "combine_warp_top_router_b200", "csrc", "route_topk.cu")


def _sort8_comparators():
    src = open(SRC).read()
    body = src[src.index("__device__ __forceinline__ void sort8("):]
    body = body[:body.index("\n}\n")]
    pairs = [(int(a), int(b)) for a, b in re.findall(r"cx\(a\[(\d)\], a\[(\d)\]\)", body)]
    return pairs


def _run(net, x):
    x = list(x)
    for i, j in net:
        if x[i] < x[j]:          # descending compare-exchange
            x[i], x[j] = x[j], x[i]
    return x


def _bitonic8(x):
    x = list(x)
    for d in (4, 2, 1):
        for i in range(8):
            if i & d == 0 and x[i] < x[i + d]:
                x[i], x[i + d] = x[i + d], x[i]
    return x


def test_sort8_has_19_comparators_and_sorts_every_01_input():
    net = _sort8_comparators()
    assert len(net) == 19
    for bits in itertools.product((0, 1), repeat=8):
        assert _run(net, bits) == sorted(bits, reverse=True), bits


def test_merge_and_kth_largest_formula():
    net = _sort8_comparators()
    rng = np.random.default_rng(0)
    for _ in range(5000):
        x = rng.integers(0, 12, 16).tolist()        # small range: many ties
        a, b = _run(net, x[:8]), _run(net, x[8:])
        top = _bitonic8([max(a[i], b[7 - i]) for i in range(8)])
        want = sorted(x, reverse=True)
        assert top == want[:8]
        for k in range(1, 9):
            # k-th largest of the union: max over i of min(a_i, b_(k-i)), 1-based,
            # with a_0 = b_0 = +inf (the kernel's threshold)
            th = max(a[k - 1], b[k - 1])
            for i in range(1, k):
                th = max(th, min(a[i - 1], b[k - i - 1]))
            assert th == want[k - 1]
