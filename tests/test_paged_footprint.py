"""Device footprint of the paged block pools (no GPU needed: the arena plan).

The 36-layer ragged workload (64 sequences with contexts uniform in
[1024, 32768], K4/V2 with K8/V4 on layers 0-3, G64, R64) sized for its
longest sequence holds 64 x 32768 token slots per layer. With pages of 16
blocks (1024 tokens) drawn from a pool, it needs only the pages its
sequences fill. The pool footprint must equal the plan's arithmetic exactly,
and the paged cache must cost about half of the contiguous one.
"""

import math

from asymmetric_bit_kv_b200 import CacheConfig
from asymmetric_bit_kv_b200 import kvq as K
from asymmetric_bit_kv_b200 import workloads as W


def _cfg(wl, **kw):
    return CacheConfig(wl.num_layers, wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, max(wl.context),
                       wl.group_k, wl.group_v, wl.residual, wl.kv_dtype, wl.k_bits, wl.v_bits, **kw)


def _record_bytes(wl, layer):
    G, D, Gv = wl.group_k, wl.head_dim, wl.group_v
    return G * D * (wl.k_bits[layer] + wl.v_bits[layer]) // 8 + 4 * D + 4 * G * D // Gv


def test_ragged_workload_pages_halve_the_footprint():
    wl = W.qwen3_8b_layers()
    G, R, P = wl.group_k, wl.residual, 16
    # blocks each sequence holds once its context is appended (lazy flush:
    # the ring keeps 1..R tokens)
    blocks = [(L - (R - ((R - L) % G) if L > R else L)) // G for L in wl.context]
    for L, nb in zip(wl.context, blocks):
        assert 0 < L - nb * G <= R
    pages = sum(math.ceil(nb / P) for nb in blocks)
    contiguous = K.required_bytes(_cfg(wl))
    paged = K.required_bytes(_cfg(wl, page_blocks=P, pool_pages=pages))
    # the difference is exactly the block records no sequence uses, less the page tables
    max_blocks = max(wl.context) // G
    max_pages = math.ceil(max_blocks / P)
    saved = sum((wl.batch * max_blocks - pages * P) * wl.num_kv_heads * _record_bytes(wl, l)
                for l in range(wl.num_layers))
    table = wl.num_layers * wl.batch * max_pages * 4
    assert abs((contiguous - paged) - (saved - table)) <= 512 * wl.num_layers * 6  # 256-byte alignment per part
    assert paged < 0.6 * contiguous, (paged / 1e9, contiguous / 1e9)
    print(f"contiguous {contiguous / 1e9:.1f} GB, paged {paged / 1e9:.1f} GB")


def test_paged_config_validation():
    wl = W.llama3_8b_gqa()
    cfg = _cfg(wl, page_blocks=4, pool_pages=0)
    lib = K.load_library()
    c, _keep = cfg.to_c()
    import ctypes
    n = ctypes.c_size_t(0)
    assert lib.kvq_cache_required_bytes(ctypes.byref(c), ctypes.byref(n)) == K.KVQ_ERR_INVALID_ARG
    assert "pool_pages" in lib.kvq_last_error().decode()
    cfg = _cfg(wl, page_blocks=-1, pool_pages=4)
    c, _keep = cfg.to_c()
    assert lib.kvq_cache_required_bytes(ctypes.byref(c), ctypes.byref(n)) == K.KVQ_ERR_INVALID_ARG
