"""The C-ABI library builds for sm_100a, loads, and exports every entry point
declared in include/moedispatch.h (no kernel is run: no GPU needed)."""
import ctypes
import os
import re

from combine_warp_top_router_b200 import binding, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "moedispatch.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(md_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("md_route_topk", "md_dispatch_layout", "md_dispatch_permute", "md_combine",
              "md_coselect_stats", "md_token_shuffle", "md_place_correlated", "md_gather_rows",
              "md_dedup_expand"):
        assert n in names


def test_library_exports_every_declared_symbol():
    path = build.build()
    h = ctypes.CDLL(path)
    missing = [n for n in _declared() if not hasattr(h, n)]
    assert not missing, missing
    # the binding declares a signature for every entry point
    assert set(_declared()) <= set(binding._SIGNATURES)


def test_host_only_calls():
    binding.lib()
    assert binding.lib().md_version() >= 100
    assert "MD_ERR_ARG" in binding.status_string(1)
    # argument checks run on the host and enqueue nothing
    L = binding.lib()
    assert L.md_route_topk(None, 4, 8, 9, 0, None, None, None) == binding.MD_ERR_ARG
    assert L.md_dispatch_layout_workspace_size(100, 8, 2, 3, 0) == 0      # T % R != 0
    assert L.md_dispatch_layout_workspace_size(96, 8, 2, 4, 1) > 0
    assert L.md_combine(None, 0, None, None, None, 4, 2, 12, 0, None, 0, None, None, None,
                        None) == binding.MD_ERR_ARG                          # H % 8 != 0
    assert L.md_token_shuffle(None, 2, None, None, 10, 8, 4, None, None, None, None, 0, None,
                              None) == binding.MD_ERR_ARG                    # T % R != 0
    assert L.md_dedup_expand(None, 0, 12, None, None, 4, 2, 8, None, None,
                             None) == binding.MD_ERR_ARG                     # H % 8 != 0


def test_layout_workspace_does_not_grow_with_tokens():
    # the layout's scratch is per CTA and per bucket, not per tile, so it is
    # the same for every T and fits the no-alloc entry point's fixed array
    L = binding.lib()
    cap = L.md_dispatch_layout_noalloc_max_scratch()
    for E, k, R, mode in ((128, 8, 16, 1), (256, 8, 64, 1), (1024, 32, 64, 1), (1024, 32, 64, 0)):
        sizes = {L.md_dispatch_layout_workspace_size(T, E, k, R, mode)
                 for T in (R, 64 * R, 1 << 16, 1 << 20, (1 << 26) // k)}
        assert len(sizes) == 1
        assert 0 < sizes.pop() <= cap
