"""CPU-side checks of the C ABI: the library loads, exports every function
include/mla.h declares, and rejects bad arguments before touching a GPU."""

import ctypes
import math
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_boundary():
    assert _declared() == sorted([
        "mla_absorb_query", "mla_cache_insert", "mla_cache_insert_fp8", "mla_combine", "mla_decode", "mla_decode_fp8",
        "mla_decode_noalloc", "mla_decode_plan",
        "mla_get_error", "mla_index_scores", "mla_merge", "mla_num_workers", "mla_plan_bytes", "mla_status_string",
        "mla_topk", "mla_unabsorb_output", "mla_workspace_bytes"])


def test_library_exports_every_declared_symbol(libmla):
    lib = ctypes.CDLL(libmla.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    assert set(_declared()) == set(libmla.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", libmla.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (mla_\w+)", out))
    assert exported == set(_declared())


def _desc(libmla, **kw):
    base = dict(batch=2, q_len=1, num_heads=128, num_pages=8, max_pages_per_seq=4)
    base.update(kw)
    return libmla.make_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(batch=-1), 1), (dict(q_len=0), 1), (dict(num_pages=0), 1), (dict(max_pages_per_seq=0), 1),
    (dict(topk=-3), 1), (dict(causal=True, topk=4), 1), (dict(softmax_scale=0.0), 1),
    (dict(softmax_scale=float("nan")), 1), (dict(softmax_scale=float("inf")), 1),
    (dict(d_latent=256), 2), (dict(d_rope=32), 2), (dict(page_size=16), 2), (dict(num_heads=0), 1),
    (dict(num_heads=129), 2), (dict(num_heads=256), 2),
])
def test_bad_descriptors_rejected_before_launch(libmla, kw, status):
    d = _desc(libmla, **kw)
    assert libmla.mla_plan_bytes(d) == 0
    assert libmla.mla_workspace_bytes(d) == 0
    assert libmla.mla_num_workers(d) == 0
    assert libmla.mla_decode_plan(d, 16, 16, 1 << 20, None) == status
    assert libmla.mla_decode(d, 16, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 30, None) == status
    assert libmla.mla_combine(d, 16, 16, 1 << 30, 16, 16, None) == status


def test_null_and_misaligned_pointers_rejected(libmla):
    d = _desc(libmla)
    INV = libmla.MLA_ERR_INVALID_ARG
    assert libmla.mla_decode_plan(d, None, 16, 1 << 20, None) == INV
    assert libmla.mla_decode_plan(d, 16, None, 1 << 20, None) == INV
    assert libmla.mla_decode_plan(d, 16, 8, 1 << 20, None) == INV            # plan not 16-B aligned
    args = [16] * 9
    for i in range(9):
        a = list(args)
        a[i] = None
        if i == 5:      # topk_indices may be NULL for a dense descriptor: that alone is not an error
            continue
        assert libmla.mla_decode(d, *a[:9], 1 << 30, None) == INV, i
    # misaligned q / cache / out
    for i in (1, 2, 6):
        a = list(args)
        a[i] = 24
        assert libmla.mla_decode(d, *a, 1 << 30, None) == INV, i
    sparse = _desc(libmla, topk=8)
    a = list(args)
    a[5] = None
    assert libmla.mla_decode(sparse, *a, 1 << 30, None) == INV
    assert libmla.mla_combine(d, None, 16, 1 << 30, 16, 16, None) == INV
    assert libmla.mla_combine(d, 16, 16, 1 << 30, 16, 18, None) == INV       # lse not 4-B aligned
    st, _ = libmla.mla_get_error(None)
    assert st == INV


def _idesc(libmla, **kw):
    base = dict(num_tokens=4, batch=2, max_pages_per_seq=4, num_pages=8, max_positions=256)
    base.update(kw)
    return libmla.make_insert_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(num_tokens=-1), 1), (dict(batch=-1), 1), (dict(max_pages_per_seq=0), 1), (dict(num_pages=0), 1),
    (dict(max_positions=0), 1), (dict(eps=-1e-6), 1), (dict(eps=float("nan")), 1), (dict(eps=float("inf")), 1),
    (dict(d_latent=256), 2), (dict(d_rope=32), 2), (dict(page_size=16), 2),
    (dict(max_pages_per_seq=(1 << 25) + 1), 2), (dict(num_pages=(1 << 25) + 1), 2),
])
def test_cache_insert_bad_descriptors_rejected(libmla, kw, status):
    d = _idesc(libmla, **kw)
    assert libmla.mla_cache_insert(d, 16, 16, 16, 16, 16, 16, 16, 16, None, None) == status


def test_cache_insert_null_misaligned_and_empty(libmla):
    d = _idesc(libmla)
    good = [16, 16, 16, 16, 16, 16, 16, 16]
    for i in range(8):
        args = list(good)
        args[i] = None
        assert libmla.mla_cache_insert(d, *args, None, None) == libmla.MLA_ERR_INVALID_ARG, i
    for i, off in ((0, 8), (1, 8), (2, 2), (3, 2), (7, 8)):
        args = list(good)
        args[i] += off
        assert libmla.mla_cache_insert(d, *args, None, None) == libmla.MLA_ERR_INVALID_ARG, i
    assert libmla.mla_cache_insert(d, *good, 18, None) == libmla.MLA_ERR_INVALID_ARG
    # no tokens: nothing to do, no pointer is read and nothing is launched
    assert libmla.mla_cache_insert(_idesc(libmla, num_tokens=0), *([None] * 8), None, None) == libmla.MLA_OK


@pytest.mark.parametrize("kw,status", [
    (dict(num_tokens=-1), 1), (dict(num_heads=0), 1), (dict(num_heads=129), 2), (dict(d_nope=64), 2),
    (dict(d_rope=32), 2), (dict(d_latent=256), 2), (dict(d_v=64), 2), (dict(num_tokens=65535 * 128 + 1), 2),
])
def test_absorb_bad_descriptors_rejected(libmla, kw, status):
    base = dict(num_tokens=4, num_heads=8)
    base.update(kw)
    d = libmla.make_absorb_desc(**base)
    assert libmla.mla_absorb_query(d, 16, 16, 16, None, None) == status
    assert libmla.mla_unabsorb_output(d, 16, 16, 16, None, None) == status


def test_absorb_null_misaligned_and_empty(libmla):
    d = libmla.make_absorb_desc(num_tokens=4, num_heads=8)
    for fn in (libmla.mla_absorb_query, libmla.mla_unabsorb_output):
        for i in range(3):
            args = [16, 16, 16]
            args[i] = None
            assert fn(d, *args, None, None) == libmla.MLA_ERR_INVALID_ARG, i
            args = [16, 16, 16]
            args[i] = 24
            assert fn(d, *args, None, None) == libmla.MLA_ERR_INVALID_ARG, i
        assert fn(d, 16, 16, 16, 18, None) == libmla.MLA_ERR_INVALID_ARG
        assert fn(libmla.make_absorb_desc(num_tokens=0, num_heads=8), None, None, None, None, None) == libmla.MLA_OK


def test_plan_too_small_rejected(libmla):
    d = _desc(libmla)
    need = libmla.mla_plan_bytes(d)
    assert need == ((8 + 2 * 2 + 1) * 4 + 15) // 16 * 16
    assert libmla.mla_decode_plan(d, 16, 16, need - 4, None) == libmla.MLA_ERR_WORKSPACE_TOO_SMALL


def test_status_strings(libmla):
    seen = set()
    for s in range(7):
        txt = libmla.mla_status_string(s)
        assert txt and txt not in seen
        seen.add(txt)
    assert libmla.mla_status_string(99) == "unknown status"


def test_binding_fails_loudly_without_library():
    env = dict(os.environ, MLA_LIB="/nonexistent/libmla.so")
    code = "import mla_latent_kv_26_b200.binding"
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env, capture_output=True, text=True)
    assert r.returncode != 0 and "libmla.so is not built" in r.stderr


# ---------------------------------------------------------------- limits checked on the host alone


@pytest.mark.parametrize("kw", [
    dict(batch=1 << 20, max_pages_per_seq=4096),                 # 2^32 pages of dense work
    dict(batch=1 << 24, max_pages_per_seq=128),                  # 2^31
    dict(batch=1 << 24, topk=256 * 64),                          # sparse: 2^24 tasks x 256 pages
])
def test_page_total_beyond_32_bits_rejected(libmla, kw):
    """The plan kernel sums every task's pages in 32-bit prefixes: a
    descriptor whose largest total reaches 2^31 is rejected up front."""
    d = _desc(libmla, **kw)
    assert libmla.mla_plan_bytes(d) == 0
    assert libmla.mla_decode_plan(d, 16, 16, 1 << 40, None) == libmla.MLA_ERR_UNSUPPORTED
    assert libmla.mla_decode_noalloc(d, 16, 16, 16, 16, 16, 16, 16, None) == libmla.MLA_ERR_UNSUPPORTED


def test_page_total_just_below_32_bits_accepted(libmla):
    d = _desc(libmla, batch=(1 << 24) - 1, max_pages_per_seq=128)   # (2^24 - 1) * 128 < 2^31
    assert libmla.mla_plan_bytes(d) > 0


def _noalloc_fits(T, H, plan_bytes):
    """The documented limit: round_up(plan, 256) + (T + 1) * H * 2056 <= 32 MiB."""
    return ((plan_bytes + 255) // 256) * 256 + (T + 1) * H * 2056 <= 32 << 20


@pytest.mark.parametrize("batch,heads", [(1 << 22, 1), (1 << 24, 1), (127, 128), (400, 128), (16256, 1),
                                         (2039, 8)])
def test_noalloc_too_large_rejected_before_the_device(libmla, batch, heads):
    """mla_decode_noalloc sizes its fixed 32 MiB scratch on the host before any
    CUDA call: a plan that alone exceeds it (4M and 16M query tokens of one
    head) or partials that do not fit give MLA_ERR_WORKSPACE_TOO_SMALL, with
    dummy pointers and no GPU."""
    d = _desc(libmla, batch=batch, num_heads=heads, max_pages_per_seq=1)
    assert not _noalloc_fits(batch, heads, libmla.mla_plan_bytes(d))
    assert libmla.mla_decode_noalloc(d, 16, 16, 16, 16, 16, 16, 16, None) == libmla.MLA_ERR_WORKSPACE_TOO_SMALL


@pytest.mark.parametrize("batch,heads", [(126, 128), (16255, 1), (2038, 8)])
def test_noalloc_largest_fitting_batch_passes_the_size_check(libmla, batch, heads):
    d = _desc(libmla, batch=batch, num_heads=heads, max_pages_per_seq=1)
    assert _noalloc_fits(batch, heads, libmla.mla_plan_bytes(d))
    assert not _noalloc_fits(batch + 1, heads, libmla.mla_plan_bytes(_desc(libmla, batch=batch + 1,
                                                                             num_heads=heads,
                                                                             max_pages_per_seq=1)))
    import torch

    if torch.cuda.is_available():
        pytest.skip("past the size check the call launches kernels; dummy pointers only without a GPU")
    st = libmla.mla_decode_noalloc(d, 16, 16, 16, 16, 16, 16, 16, None)
    assert st == libmla.MLA_ERR_CUDA        # reached the device set-up: no GPU here


# ---------------------------------------------------------------- indexer and top-k


@pytest.mark.parametrize("kw,status", [
    (dict(batch=-1), 1), (dict(q_len=0), 1), (dict(num_heads=0), 1), (dict(num_keys=-1), 1),
    (dict(head_dim=64), 2), (dict(num_heads=24), 2), (dict(num_heads=272), 2),
    (dict(batch=1 << 16, num_keys=1 << 16), 2), (dict(batch=1 << 12, q_len=1 << 12, num_heads=256), 2),
])
def test_index_bad_descriptors_rejected(libmla, kw, status):
    base = dict(batch=2, q_len=1, num_heads=64, num_keys=300)
    base.update(kw)
    d = libmla.make_index_desc(**base)
    assert libmla.mla_index_scores(d, 16, 16, 16, 16, 16, None, None) == status


def test_index_null_misaligned_and_empty(libmla):
    d = libmla.make_index_desc(batch=2, q_len=1, num_heads=64, num_keys=300)
    good = [16, 16, 16, 16, 16]
    for i in range(5):
        a = list(good)
        a[i] = None
        assert libmla.mla_index_scores(d, *a, None, None) == libmla.MLA_ERR_INVALID_ARG, i
    for i, off in ((0, 8), (1, 4), (2, 8), (3, 2), (4, 2)):
        a = list(good)
        a[i] += off
        assert libmla.mla_index_scores(d, *a, None, None) == libmla.MLA_ERR_INVALID_ARG, i
    assert libmla.mla_index_scores(d, *good, 18, None) == libmla.MLA_ERR_INVALID_ARG
    for empty in (dict(batch=0), dict(num_keys=0)):
        e = libmla.make_index_desc(**dict(dict(batch=2, q_len=1, num_heads=64, num_keys=300), **empty))
        assert libmla.mla_index_scores(e, None, None, None, None, None, None, None) == libmla.MLA_OK


def test_topk_bad_arguments_rejected(libmla):
    INV = libmla.MLA_ERR_INVALID_ARG
    mk = libmla.make_topk_desc
    assert libmla.mla_topk(mk(rows=-1, num_keys=8, k=2), 16, None, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=-1, k=2), 16, None, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=0), 16, None, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=2), None, None, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=2), 16, None, None, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=2), 18, None, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=2), 16, 18, 16, None) == INV
    assert libmla.mla_topk(mk(rows=2, num_keys=8, k=2), 16, None, 18, None) == INV
    assert libmla.mla_topk(mk(rows=1 << 29, num_keys=8, k=2), 16, None, 16, None) == libmla.MLA_ERR_UNSUPPORTED
    assert libmla.mla_topk(mk(rows=0, num_keys=8, k=2), None, None, None, None) == libmla.MLA_OK


def test_merge_bad_arguments_rejected(libmla):
    INV = libmla.MLA_ERR_INVALID_ARG
    mk = libmla.make_merge_desc
    assert libmla.mla_merge(mk(parts=0, rows=4), 16, 16, 16, 16, None) == INV
    assert libmla.mla_merge(mk(parts=2, rows=-1), 16, 16, 16, 16, None) == INV
    assert libmla.mla_merge(mk(parts=2, rows=4, d_latent=256), 16, 16, 16, 16, None) == libmla.MLA_ERR_UNSUPPORTED
    for i in range(4):
        a = [16, 16, 16, 16]
        a[i] = None
        assert libmla.mla_merge(mk(parts=2, rows=4), *a, None) == INV, i
    for i, off in ((0, 8), (1, 2), (2, 8), (3, 2)):
        a = [16, 16, 16, 16]
        a[i] += off
        assert libmla.mla_merge(mk(parts=2, rows=4), *a, None) == INV, i
    assert libmla.mla_merge(mk(parts=2, rows=0), None, None, None, None, None) == libmla.MLA_OK


def test_fp8_entries_validate_like_their_bf16_counterparts(libmla):
    """mla_decode_fp8 and mla_cache_insert_fp8 share the argument checks of
    mla_decode and mla_cache_insert (rejected before any launch)."""
    for kw, status in [(dict(batch=-1), 1), (dict(d_latent=256), 2), (dict(num_heads=129), 2),
                       (dict(causal=True, topk=4), 1)]:
        d = _desc(libmla, **kw)
        assert libmla.mla_decode_fp8(d, 16, 16, 16, 16, 16, 16, 16, 16, 16, 1 << 30, None) == status
    d = _desc(libmla)
    args = [16] * 9
    for i in range(9):
        if i == 5:
            continue
        a = list(args)
        a[i] = None
        assert libmla.mla_decode_fp8(d, *a, 1 << 30, None) == libmla.MLA_ERR_INVALID_ARG, i
    for kw, status in [(dict(num_tokens=-1), 1), (dict(eps=-1.0), 1), (dict(d_latent=256), 2)]:
        assert libmla.mla_cache_insert_fp8(_idesc(libmla, **kw), 16, 16, 16, 16, 16, 16, 16, 16, None, None) == status
    assert libmla.mla_cache_insert_fp8(_idesc(libmla), 16, 16, 16, 16, 16, 16, 16, 24, None, None) == \
        libmla.MLA_ERR_INVALID_ARG
