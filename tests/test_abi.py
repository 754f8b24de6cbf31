"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, sizes arenas by the closed form, and rejects bad arguments on
the host before touching the device."""

import ctypes
import os
import re

import pytest
import torch

from asymmetric_bit_kv_b200 import CacheConfig, KvqError, load_library, required_bytes
from asymmetric_bit_kv_b200 import kvq as K
from oracle import kvq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^KVQ_API\s+[\w\s\*]+?\b(kvq_\w+)\s*\(", src, flags=re.M))
    return names


def test_header_declares_entry_points():
    names = _declared()
    for n in ["kvq_cache_create", "kvq_append", "kvq_flush_residual", "kvq_decode_attention", "kvq_dequant"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = load_library()
    for name in sorted(_declared()):
        assert hasattr(lib, name), name


def test_status_strings():
    lib = load_library()
    assert lib.kvq_status_string(0) == b"ok"
    assert lib.kvq_status_string(-3) == b"sequence capacity exceeded"


def _cfg(**kw):
    base = dict(num_layers=1, max_batch=4, num_q_heads=8, num_kv_heads=2, head_dim=128, max_tokens=4096,
                group_k=64, group_v=64, residual=128, kv_dtype=torch.bfloat16, k_bits=[2], v_bits=[4])
    base.update(kw)
    return CacheConfig(**base)


def test_required_bytes_covers_the_packed_cache():
    cfg = _cfg()
    n = required_bytes(cfg)
    per_tok = O.quantized_bytes_per_token(2, 128, 2, 4, 64, 64)
    packed = per_tok * cfg.max_batch * (cfg.max_tokens // cfg.group_k) * cfg.group_k
    ring = 2 * cfg.max_batch * 2 * cfg.residual * 128 * 2
    assert n >= packed + ring
    assert n < (packed + ring) * 1.5 + (1 << 24)   # plus lengths and split workspace


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=64), K.KVQ_ERR_UNSUPPORTED),
    (dict(group_k=48), K.KVQ_ERR_UNSUPPORTED),
    (dict(group_v=256), K.KVQ_ERR_UNSUPPORTED),
    (dict(residual=96), K.KVQ_ERR_INVALID_ARG),
    (dict(num_q_heads=7), K.KVQ_ERR_INVALID_ARG),
    (dict(num_q_heads=6), K.KVQ_ERR_UNSUPPORTED),
    (dict(num_q_heads=32), K.KVQ_ERR_UNSUPPORTED),
    (dict(k_bits=[3]), K.KVQ_ERR_UNSUPPORTED),
    (dict(max_batch=0), K.KVQ_ERR_INVALID_ARG),
    (dict(max_batch=513), K.KVQ_ERR_INVALID_ARG),
    (dict(kv_dtype=torch.float32), K.KVQ_ERR_UNSUPPORTED),
])
def test_invalid_configs(kw, status):
    with pytest.raises(KvqError) as e:
        required_bytes(_cfg(**kw))
    assert e.value.status == status


def test_create_rejects_bad_arena_on_host():
    lib = load_library()
    cfg = _cfg()
    c, _keep = cfg.to_c()
    h = ctypes.c_void_p()
    n = required_bytes(cfg)
    assert lib.kvq_cache_create(ctypes.byref(c), None, n, ctypes.byref(h)) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_cache_create(ctypes.byref(c), 0x1000010, n, ctypes.byref(h)) == K.KVQ_ERR_INVALID_ARG
    assert lib.kvq_cache_create(ctypes.byref(c), 0x1000000, n - 1, ctypes.byref(h)) == K.KVQ_ERR_WORKSPACE
    assert b"required" in lib.kvq_last_error()
    assert lib.kvq_append(None, 0, None, None, None, 0, None) == K.KVQ_ERR_INVALID_ARG
    count = ctypes.c_uint64(7)
    assert lib.kvq_cache_kernel_launches(None, ctypes.byref(count)) == K.KVQ_ERR_INVALID_ARG
    assert count.value == 7
    assert lib.kvq_decode_attention(None, 0, None, None, 0, 1.0, 1, None) == K.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("kb,vb,G,Gv,k_axis", [
    (2, 4, 64, 64, 0), (2, 2, 32, 32, 0), (4, 2, 128, 64, 0), (8, 8, 64, 128, 0),
    (2, 2, 64, 128, 1), (4, 4, 32, 64, 1), (8, 2, 128, 32, 1),
])
def test_block_record_bytes_match_the_closed_form(kb, vb, G, Gv, k_axis):
    # one more run of 16 blocks per sequence grows the arena by exactly that
    # many block records per (sequence, KV head, layer); a record holds G
    # tokens at the closed-form bytes per token (KV1 card, Memory: codes plus
    # an fp16 scale and zero point per group)
    def cfg(max_tokens, **kw):
        return CacheConfig(2, 3, 8, 2, 128, max_tokens, G, Gv, 128, torch.bfloat16, [kb] * 2, [vb] * 2,
                           k_axis=[k_axis] * 2, **kw)
    m = 200 * G  # large enough that the split workspace no longer grows
    grow = required_bytes(cfg(m + 16 * G)) - required_bytes(cfg(m))
    per_head_token = O.quantized_bytes_per_token(1, 128, kb, vb, G, Gv, k_axis=k_axis)
    assert grow == 2 * 3 * 2 * 16 * G * per_head_token
    # a paged layer: one more page of 4 blocks per layer, for every KV head
    paged = [required_bytes(cfg(m, page_blocks=4, pool_pages=p)) for p in (10, 11)]
    assert paged[1] - paged[0] == 2 * 2 * 4 * G * per_head_token
