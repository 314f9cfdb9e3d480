"""The C ABI library loads without a GPU, exports every function include/*.h
declares, and rejects bad arguments on the host (nothing is enqueued, so these
run on a machine without a GPU)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

HEADERS = [os.path.join(ROOT, "include", f) for f in sorted(os.listdir(os.path.join(ROOT, "include")))
           if f.endswith(".h")]

OK, ENULL, ESHAPE, EDTYPE, EUNSUP, EWS, ECUDA, EALIGN = 0, -1, -2, -3, -4, -5, -6, -7
F32, F16, BF16, FP8 = 0, 1, 2, 3
A = 1 << 20          # a fake, 256-byte aligned "device" address; never dereferenced


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_367_b200 import build
    build.build()
    import paged_kv_cache_367_b200 as pkv
    return pkv.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*([a-z_0-9]+)\s*\(",
                                text, flags=re.M))
    return sorted(names)


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert {"paged_kv_append", "paged_attention_decode", "paged_attention_workspace_size",
            "pkv_status_string", "pkv_version", "pkv_bm_create", "paged_kv_copy_blocks",
            "paged_kv_swap_blocks"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_binding_names_match_the_header(lib):
    import paged_kv_cache_367_b200 as pkv
    from paged_kv_cache_367_b200.blocks import BlockManager
    assert set(pkv.EXPORTED_SYMBOLS) == set(declared_functions())
    # pkv_bm_<name> is BlockManager.<name> (create / destroy: construction / close).
    special = {"create": "__init__", "destroy": "close"}
    for n in pkv.EXPORTED_SYMBOLS:
        if n.startswith("pkv_bm_"):
            m = n[len("pkv_bm_"):]
            assert hasattr(BlockManager, special.get(m, m)), n
        else:
            assert callable(getattr(pkv, n)), n


def test_status_strings(lib):
    for s in (OK, ENULL, ESHAPE, EDTYPE, EUNSUP, EWS, ECUDA, EALIGN, -8, -9, -10):
        assert lib.pkv_status_string(s)
    assert lib.pkv_status_string(12345) == b"unknown status"
    assert lib.pkv_version() >= 100


def decode(lib, **kw):
    a = dict(out=A, query=A, k_cache=A, v_cache=A, block_table=A, seq_lens=A, num_seqs=4,
             num_heads=8, num_kv_heads=2, head_dim=128, block_size=16, max_blocks_per_seq=8,
             num_blocks=100, max_seq_len=128, scale=0.1, q_dtype=BF16, cache_dtype=BF16,
             k_scale=A, v_scale=A, partition_size=0, max_ctas=0, flags=0, workspace=None,
             workspace_bytes=0, stream=None)
    a.update(kw)
    return lib.paged_attention_decode(*a.values())


def append(lib, **kw):
    a = dict(key=A, value=A, k_cache=A, v_cache=A, slot_mapping=A, num_tokens=4, num_kv_heads=2,
             head_dim=128, block_size=16, num_blocks=10, src_dtype=BF16, cache_dtype=BF16,
             k_scale=A, v_scale=A, stream=None)
    a.update(kw)
    return lib.paged_kv_append(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(out=None), ENULL), (dict(query=None), ENULL), (dict(block_table=None), ENULL),
    (dict(seq_lens=None), ENULL), (dict(cache_dtype=FP8, k_scale=None), ENULL),
    (dict(num_heads=6, num_kv_heads=4), ESHAPE), (dict(num_kv_heads=0), ESHAPE),
    (dict(num_seqs=-1), ESHAPE), (dict(max_seq_len=-1), ESHAPE), (dict(num_blocks=0), ESHAPE),
    (dict(max_blocks_per_seq=0), ESHAPE), (dict(partition_size=-16), ESHAPE),
    (dict(partition_size=24), ESHAPE), (dict(max_ctas=-1), ESHAPE),
    (dict(scale=float("nan")), ESHAPE), (dict(scale=float("inf")), ESHAPE),
    (dict(head_dim=96), EUNSUP), (dict(head_dim=256), EUNSUP), (dict(block_size=4), EUNSUP),
    (dict(block_size=64), EUNSUP), (dict(q_dtype=FP8, cache_dtype=FP8), EDTYPE),
    (dict(q_dtype=7), EDTYPE), (dict(q_dtype=BF16, cache_dtype=F16), EDTYPE),
    (dict(out=A + 8), EALIGN), (dict(k_cache=A + 4), EALIGN), (dict(seq_lens=A + 2), EALIGN),
    (dict(partition_size=512, max_seq_len=1000), EWS),
    (dict(partition_size=512, max_seq_len=1000, workspace=A, workspace_bytes=100), EWS),
    (dict(num_seqs=0, out=None), OK),
])
def test_decode_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert decode(lib, **kw) == code


def test_workspace_size(lib):
    ws = lib.paged_attention_workspace_size
    assert ws(4, 8, 2, 128, 128, 0) == 0
    assert ws(4, 8, 2, 128, 512, 512) == 0          # nothing can be cut
    need = ws(4, 8, 2, 128, 1000, 512)
    g = 8 // 2
    assert need >= 2 * 1024 * g * (128 + 1) * 4 + 4 * 2 * 4   # two slots per CTA + counters
    assert need % 256 == 0
    assert ws(4, 8, 2, 128, 100000, 512) == need     # independent of max_seq_len
    assert ws(-1, 8, 2, 128, 1000, 512) == 0
    assert decode(lib, partition_size=512, max_seq_len=1000, workspace=A + 256,
                  workspace_bytes=need - 1) == EWS
    assert decode(lib, partition_size=512, max_seq_len=1000, workspace=A + 16,
                  workspace_bytes=need) == EALIGN


@pytest.mark.parametrize("kw,code", [
    (dict(key=None), ENULL), (dict(slot_mapping=None), ENULL),
    (dict(cache_dtype=FP8, v_scale=None), ENULL), (dict(num_tokens=-1), ESHAPE),
    (dict(head_dim=100), ESHAPE), (dict(num_kv_heads=0), ESHAPE), (dict(block_size=0), ESHAPE),
    (dict(num_blocks=0), ESHAPE), (dict(src_dtype=FP8, cache_dtype=FP8), EDTYPE),
    (dict(src_dtype=F32, cache_dtype=BF16), EDTYPE), (dict(key=A + 8), EALIGN),
    (dict(slot_mapping=A + 4), EALIGN), (dict(num_tokens=0, key=None), OK),
])
def test_append_rejects_bad_arguments_on_the_host(lib, kw, code):
    assert append(lib, **kw) == code


def test_binding_raises_when_the_library_is_missing(tmp_path):
    import paged_kv_cache_367_b200 as pkv
    saved = pkv._lib
    pkv._lib = None
    try:
        with pytest.raises(ImportError):
            pkv.load_library(str(tmp_path / "absent.so"))
    finally:
        pkv._lib = saved


def copy(lib, **kw):
    a = dict(k_cache=A, v_cache=A, block_mapping=A, num_pairs=4, block_bytes=4096,
             num_blocks=100, stream=None)
    a.update(kw)
    return lib.paged_kv_copy_blocks(*a.values())


def swap(lib, **kw):
    a = dict(src_k=A, src_v=A, dst_k=A, dst_v=A, block_mapping=A, num_pairs=4, block_bytes=4096,
             src_num_blocks=100, dst_num_blocks=10, stream=None)
    a.update(kw)
    return lib.paged_kv_swap_blocks(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(num_pairs=0), OK), (dict(num_pairs=0, k_cache=None), OK),
    (dict(k_cache=None), ENULL), (dict(block_mapping=None), ENULL),
    (dict(num_pairs=-1), ESHAPE), (dict(block_bytes=0), ESHAPE), (dict(block_bytes=4100), ESHAPE),
    (dict(num_blocks=-1), ESHAPE), (dict(v_cache=A + 8), EALIGN), (dict(block_mapping=A + 4), EALIGN),
])
def test_copy_blocks_rejects_bad_arguments(lib, kw, code):
    assert copy(lib, **kw) == code


@pytest.mark.parametrize("kw,code", [
    (dict(num_pairs=0), OK), (dict(dst_k=None), ENULL), (dict(src_v=None), ENULL),
    (dict(block_bytes=8), ESHAPE), (dict(dst_num_blocks=-2), ESHAPE), (dict(src_k=A + 1), EALIGN),
])
def test_swap_blocks_rejects_bad_arguments(lib, kw, code):
    assert swap(lib, **kw) == code


def prefill(lib, **kw):
    a = dict(out=A, query=A, k_cache=A, v_cache=A, block_table=A, seq_lens=A, query_start=A,
             num_seqs=2, num_q_tokens=10, max_q_len=8, num_heads=8, num_kv_heads=2, head_dim=128,
             block_size=16, max_blocks_per_seq=8, num_blocks=100, scale=0.1, q_dtype=BF16,
             cache_dtype=BF16, k_scale=A, v_scale=A, flags=0, stream=None)
    a.update(kw)
    return lib.paged_attention_prefill(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(num_seqs=0), OK), (dict(num_q_tokens=0), OK), (dict(max_q_len=0), OK),
    (dict(out=None), ENULL), (dict(query_start=None), ENULL), (dict(block_table=None), ENULL),
    (dict(num_heads=6, num_kv_heads=4), ESHAPE), (dict(num_seqs=-1), ESHAPE),
    (dict(num_blocks=0), ESHAPE), (dict(max_blocks_per_seq=0), ESHAPE),
    (dict(scale=float("nan")), ESHAPE), (dict(num_seqs=70000), ESHAPE),
    (dict(head_dim=96), EUNSUP), (dict(block_size=4), EUNSUP),
    (dict(q_dtype=F32, cache_dtype=F32), EDTYPE), (dict(q_dtype=F32, cache_dtype=FP8), EDTYPE),
    (dict(cache_dtype=F16), EDTYPE), (dict(cache_dtype=FP8, k_scale=None), ENULL),
    (dict(cache_dtype=FP8, v_scale=None), ENULL),
    (dict(query=A + 8), EALIGN), (dict(query_start=A + 2), EALIGN), (dict(flags=2), ESHAPE),
])
def test_prefill_rejects_bad_arguments(lib, kw, code):
    assert prefill(lib, **kw) == code


def test_decode_rejects_unknown_flags(lib):
    assert decode(lib, flags=32) == ESHAPE
    assert decode(lib, flags=1 << 31) == ESHAPE
    assert decode(lib, flags=8 | 16) == ESHAPE          # tensor cores and CUDA cores at once


def test_marshalled_argument_lists_match_the_c_signatures(lib):
    """append_args / decode_args give one value per C parameter, each one its
    declared ctypes type accepts, with the sizes in their places; a decode call
    made with them on an empty batch succeeds without touching the GPU."""
    import torch
    import paged_kv_cache_367_b200 as pkv
    key = torch.zeros(3, 2, 64, dtype=torch.bfloat16)
    pool = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    slots = torch.full((3,), -1, dtype=torch.int64)
    a = pkv.append_args(key, key, pool, pool, slots, stream=0)
    assert len(a) == len(lib.paged_kv_append.argtypes)
    conv = [t(x) for t, x in zip(lib.paged_kv_append.argtypes, a)]
    assert [c.value for c in conv[5:10]] == [3, 2, 64, 16, 4]
    q = torch.zeros(0, 4, 64, dtype=torch.bfloat16)
    bt = torch.zeros(0, 1, dtype=torch.int32)
    ln = torch.zeros(0, dtype=torch.int32)
    d = pkv.decode_args(q, q, pool, pool, bt, ln, max_seq_len=0, scale=0.125, stream=0)
    assert len(d) == len(lib.paged_attention_decode.argtypes)
    conv = [t(x) for t, x in zip(lib.paged_attention_decode.argtypes, d)]
    assert [c.value for c in conv[6:13]] == [0, 4, 2, 64, 16, 1, 4]
    assert lib.paged_attention_decode(*conv) == OK
