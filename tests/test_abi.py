"""The C-ABI library builds, loads and exports every symbol include/msa.h declares; host-only
argument validation of msa_plan_create (no GPU needed: plan creation does no device work)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "msa.h")).read()
    return sorted(set(re.findall(r"^(?:msa_status|void|size_t|uint64_t|const char\*)\s+(msa_\w+)\(", src, re.M)))


def test_library_exports_every_declared_symbol():
    from dynamic_sparse_attention_head_b200 import build
    lib = ctypes.CDLL(build.build())
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), f"libmsa.so does not export {n}"


def test_binding_names_match_header():
    import dynamic_sparse_attention_head_b200 as msa
    assert sorted(msa.EXPORTS) == _declared()


def test_plan_validation_is_host_only():
    import dynamic_sparse_attention_head_b200 as msa
    from workload import TEXT, Head, Problem, llama3_8b_text

    p = msa.Plan(llama3_8b_text(L=4096))
    assert p.workspace_bytes > 0

    class Bad:
        pass

    def prob(**kw):
        b = Bad()
        b.L, b.Hq, b.Hkv, b.d, b.scale = 1024, 2, 1, 128, 0.088
        b.segments = [(0, 1024, TEXT)]
        b.heads = [Head("dense")] * 2
        for k, v in kw.items():
            setattr(b, k, v)
        return b

    for kw, code in ((dict(L=1000, segments=[(0, 1000, TEXT)]), 2), (dict(d=64), 2), (dict(Hkv=3), 2),
                     (dict(segments=[(0, 512, TEXT)]), 2), (dict(heads=[Head("vslash")] * 2), 1),
                     (dict(heads=[Head("grid")] * 2), 1), (dict(scale=0.0), 1)):
        with pytest.raises(msa.MsaError) as e:
            msa.Plan(prob(**kw))
        assert e.value.code == code, kw


def test_workspace_grows_with_length():
    import dynamic_sparse_attention_head_b200 as msa
    from workload import llama3_8b_text
    a = msa.Plan(llama3_8b_text(L=4096)).workspace_bytes
    b = msa.Plan(llama3_8b_text(L=8192)).workspace_bytes
    assert b > a


def test_indexed_workspace_drops_the_permuted_copies():
    """The index-based path's workspace is the three-call layout without its trailing permuted
    Q ([n_qslices][LP][128] bf16, at least one slice) and O ([Hq][LP][128] bf16) copies."""
    import dynamic_sparse_attention_head_b200 as msa
    import workload
    for p in (workload.llama3_8b_text(L=4096), workload.qwen2_7b_video_128k()):
        plan = msa.Plan(p)
        assert plan.workspace_bytes_indexed < plan.workspace_bytes
        assert plan.workspace_bytes - plan.workspace_bytes_indexed >= (p.Hq + 1) * p.L * 128 * 2
        assert plan.workspace_bytes_indexed % 256 == 0


def test_attention_units_chunking_rule(monkeypatch):
    """Keys are chunked (131072 per chunk) only when one head's K and V exceed ~96 MB; the
    environment override applies at plan creation."""
    import dynamic_sparse_attention_head_b200 as msa
    import workload
    monkeypatch.delenv("MSA_ATTN_CHUNK_KEYS", raising=False)
    assert msa.Plan(workload.qwen2_7b_video_128k()).attention_units()[1] == 1
    units, chunks = msa.Plan(workload.longvila_1m()).attention_units()
    assert chunks == 8
    # the threshold: K and V of one head above 96 MB (L x 512 B), i.e. L > 196608
    assert msa.Plan(workload.llama3_8b_text(L=196608)).attention_units()[1] == 1
    assert msa.Plan(workload.llama3_8b_text(L=196672)).attention_units()[1] == 2
    assert msa.Plan(workload.llama3_8b_text(L=262144)).attention_units()[1] == 2
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "256")
    p = workload.llama3_8b_text(L=2048)
    assert msa.Plan(p).attention_units()[1] == 8
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "0")
    units, chunks = msa.Plan(p).attention_units()
    assert chunks == 1


def test_unit_band_overrides(monkeypatch):
    """Unit bands exist only over chunked keys; the band-size overrides apply at plan creation
    and only change how the units are grouped, not how many there are."""
    import dynamic_sparse_attention_head_b200 as msa
    import workload
    p = workload.llama3_8b_text(L=2048)
    monkeypatch.delenv("MSA_ATTN_BAND_SLOTS", raising=False)
    monkeypatch.delenv("MSA_ATTN_MIN_BAND_UNITS", raising=False)
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "0")
    assert msa.Plan(p).attention_work()[2] == 0
    monkeypatch.setenv("MSA_ATTN_CHUNK_KEYS", "256")
    units, chunks, bands = msa.Plan(p).attention_work()
    assert chunks == 8 and bands >= 1
    monkeypatch.setenv("MSA_ATTN_BAND_SLOTS", "1")
    monkeypatch.setenv("MSA_ATTN_MIN_BAND_UNITS", "1")
    units2, chunks2, bands2 = msa.Plan(p).attention_work()
    assert (units2, chunks2) == (units, chunks) and bands2 > bands
    items = units // chunks
    assert bands2 <= items


def test_workspace_size_and_state_checks_come_before_any_device_access():
    """The size, alignment and call-order checks of the calls return before anything touches
    device memory, so they are exercised here with placeholder addresses (never dereferenced)."""
    import ctypes
    import dynamic_sparse_attention_head_b200 as msa
    from dynamic_sparse_attention_head_b200 import _lib, Strides
    from workload import llama3_8b_text

    plan = msa.Plan(llama3_8b_text(L=4096))
    full, indexed = plan.workspace_bytes, plan.workspace_bytes_indexed
    assert indexed < full
    ws, q, k, v, o = 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20  # aligned placeholders
    s = Strides()
    for name in ("q", "k", "v", "o"):
        setattr(s, f"{name}_head", 4096 * 128)
        setattr(s, f"{name}_row", 128)
    sp = ctypes.byref(s)
    WORKSPACE, ALIGN, STATE = 4, 3, 9
    # the index-based path needs only its own size; the three-call path the full one
    assert _lib.msa_estimate(plan._h, q, k, sp, ws, indexed - 256, None) == WORKSPACE
    assert _lib.msa_sparse_prefill_indexed(plan._h, q, k, v, o, sp, ws, indexed - 256, None, None) == WORKSPACE
    assert _lib.msa_permute(plan._h, q, k, v, sp, ws, indexed, None) == WORKSPACE
    assert _lib.msa_sparse_prefill(plan._h, q, k, v, sp, ws, indexed, None, None) == WORKSPACE
    assert _lib.msa_unpermute(plan._h, ws, indexed, o, sp, None) == WORKSPACE
    # alignment
    assert _lib.msa_sparse_prefill_indexed(plan._h, q, k, v, o, sp, ws + 128, indexed, None, None) == ALIGN
    assert _lib.msa_sparse_prefill_indexed(plan._h, q, k, v, o + 8, sp, ws, indexed, None, None) == ALIGN
    # no indices in this workspace yet: the prefill and the pair count refuse it
    assert _lib.msa_sparse_prefill_indexed(plan._h, q, k, v, o, sp, ws, indexed, None, None) == STATE
    counts = (ctypes.c_int64 * plan.problem.Hq)()
    assert _lib.msa_mask_pairs(plan._h, ws, None, None) == 1  # no output buffer
    assert _lib.msa_mask_pairs(plan._h, ws, ctypes.cast(counts, ctypes.c_void_p), None) == STATE
    # the self-test's limit is bounded to (0, 1 s]
    assert _lib.msa_selftest_timeout(plan._h, ws, 0, None) == 1
    assert _lib.msa_selftest_timeout(plan._h, ws, 2000000, None) == 1


def test_per_segment_flag_validation_and_slice_rows():
    """The per-segment option is a Q-boundary flag only; a head with one class per segment gets a
    permuted Q/O slice long enough for every segment rounded up to 128 rows."""
    import dataclasses
    import dynamic_sparse_attention_head_b200 as msa
    from workload import TEXT, VIDEO, Head, Problem
    segs = [(0, 64, TEXT), (64, 64, VIDEO)] * 8  # 16 segments of 64 tokens: 8K rows once rounded up
    segs = [(i * 64, 64, m) for i, (_, _, m) in enumerate(segs)]
    p = Problem(L=1024, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=8, k_s=8)])
    base = msa.Plan(p).workspace_bytes
    q = dataclasses.replace(p, heads=[Head("qbound", k_v=8, k_s=8, per_segment=True)])
    assert msa.Plan(q).workspace_bytes > base
    bad = msa.HeadCfg()
    bad.kind, bad.k_v, bad.k_s, bad.flags = msa.KINDS["vslash"], 8, 8, msa.HEAD_PER_SEGMENT
    import pytest
    with pytest.raises(msa.MsaError) as e:
        _plan_with_cfg(p, bad)
    assert e.value.code == 1
    ok = msa.HeadCfg()
    ok.kind, ok.k_v, ok.k_s, ok.flags = msa.KINDS["qbound"], 8, 8, msa.HEAD_PER_SEGMENT
    _plan_with_cfg(p, ok)


def _plan_with_cfg(p, cfg):
    """msa_plan_create on problem p with its heads replaced by the raw configuration cfg."""
    import ctypes
    import dynamic_sparse_attention_head_b200 as msa
    segs = (msa.Segment * len(p.segments))()
    for i, (s, n, m) in enumerate(p.segments):
        segs[i].start, segs[i].len, segs[i].modality = s, n, m
    heads = (msa.HeadCfg * p.Hq)(*([cfg] * p.Hq))
    pc = msa.ProblemC(L=p.L, Hq=p.Hq, Hkv=p.Hkv, d=p.d, scale=p.scale, n_segments=len(p.segments),
                      segments=ctypes.cast(segs, ctypes.c_void_p), heads=ctypes.cast(heads, ctypes.c_void_p))
    h = ctypes.c_void_p()
    msa._check("msa_plan_create", msa._lib.msa_plan_create(ctypes.byref(pc), ctypes.byref(h)))
    msa._lib.msa_plan_destroy(h)


def test_weight_share_argument_checks_come_before_any_device_access():
    """msa_weight_share validates its arguments on the host (placeholder addresses, never
    dereferenced) and returns at once for an empty sample."""
    import ctypes
    import dynamic_sparse_attention_head_b200 as msa
    from dynamic_sparse_attention_head_b200 import Strides, _lib
    s = Strides(q_head=131072 * 128, q_row=128, k_head=131072 * 128, k_row=128)
    fake = 1 << 20  # 16-byte aligned, never touched
    call = lambda Q=fake, K=fake, L=4096, Hq=4, Hkv=2, strides=ctypes.byref(s), scale=0.088, n=1, recall=0.95: \
        _lib.msa_weight_share(Q, K, L, Hq, Hkv, strides, scale, fake, fake, n, recall, fake, None)  # noqa: E731
    assert call(Q=None) == 1
    assert call(recall=0.0) == 1 and call(recall=1.5) == 1
    assert call(scale=0.0) == 1
    assert call(n=-1) == 1
    assert call(Hq=3) == 2  # Hq not a multiple of Hkv
    assert call(Q=fake + 8) == 3  # misaligned
    bad = Strides(q_head=131072 * 128, q_row=100, k_head=131072 * 128, k_row=128)
    assert call(strides=ctypes.byref(bad)) == 3
    assert call(n=0) == 0  # nothing to do: no launch


def test_estimation_rows_spanning_more_than_4096_positions_are_refused():
    """The last 64 text queries of 4-token text runs between 316-token video runs span 4803
    positions, above the 4096 the sweep's slash ring supports: plan creation says so."""
    import numpy as np

    import dynamic_sparse_attention_head_b200 as msa
    from workload import TEXT, VIDEO, Head, Problem
    segs, t = [], 0
    for _ in range(17):
        segs += [(t, 4, TEXT), (t + 4, 316, VIDEO)]
        t += 320
    p = Problem(L=t, Hq=1, Hkv=1, segments=segs, heads=[Head("qbound", k_v=8, k_s=16)], name="too-wide")
    rows = np.nonzero(p.modality() == TEXT)[0][-64:]
    assert rows[-1] - rows[0] > 4096
    with pytest.raises(msa.MsaError) as e:
        msa.Plan(p)
    assert e.value.code == 5  # MSA_ERR_UNSUPPORTED
    # a vertical-slash head on the same layout estimates from the last 64 positions (consecutive)
    q = Problem(L=t, Hq=1, Hkv=1, segments=segs, heads=[Head("vslash", k_v=8, k_s=16)], name="vslash-only")
    msa.Plan(q)
