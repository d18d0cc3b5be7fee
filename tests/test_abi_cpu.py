"""The C-ABI library builds, loads without a GPU and exports every symbol
that include/fp8attn.h declares; host-only entry points (selector parser,
status strings, sizes, argument checks) work on the CPU."""
import ctypes
import json
import os
import re

import numpy as np
import pytest
import torch

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "fp8attn.h")


@pytest.fixture(scope="module")
def L():
    from quantization_amax_reduce_b200 import build
    build.build()
    import quantization_amax_reduce_b200 as qar
    return qar.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(fp8attn_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 20
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings_and_sizes(L):
    assert L.fp8attn_status_string(0) == b"ok"
    assert L.fp8attn_status_string(6) == b"inconsistent cu_seqlens"
    assert L.fp8attn_ring_length() == 16
    assert L.fp8attn_workspace_bytes(0) == 0
    assert L.fp8attn_workspace_bytes(24) == 256 + 24 * 320


def test_selector_parser_golden(L, golden_dir):
    import quantization_amax_reduce_b200 as qar
    g = json.load(open(os.path.join(golden_dir, "selectors.json")))
    for c in g["cases"]:
        assert qar.parse_selector(c["text"], c["max_index"]) == set(c["expect"])
    for c in g["invalid"]:
        with pytest.raises(qar.FP8AttnError):
            qar.parse_selector(c["text"], c["max_index"])
    assert qar.parse_selector(None, 4) == set()
    assert qar.parse_selector("  ", 4) == set()
    assert qar.parse_selector(" 1 , 3 - 4 ", 5) == {1, 3, 4}


def test_selector_parser_agrees_with_oracle_on_random_strings(L):
    import oracle
    import quantization_amax_reduce_b200 as qar
    rng = np.random.Generator(np.random.PCG64(3))
    alphabet = list("0123456789,- ")
    for _ in range(3000):
        s = "".join(rng.choice(alphabet, size=rng.integers(0, 9)))
        try:
            want = oracle.parse_selector(s, 30)
        except ValueError:
            want = None
        try:
            got = qar.parse_selector(s, 30)
        except qar.FP8AttnError:
            got = None
        assert got == want, repr(s)


def test_host_argument_checks_need_no_gpu(L):
    P = ctypes.c_void_p
    # null context / bad layer are rejected before any CUDA call
    assert L.fp8attn_quantize_qkv(None, 0, 0, P(16), P(16), P(16), 1024, 128, None, P(16), 1,
                                  8, 8, 8, 128, P(16), P(16), P(16), None) == 1
    # head_dim other than 128 is unsupported
    assert L.fp8attn_varlen_fwd(P(16), P(16), P(16), P(16), 1, 8, 8, 8, 64, P(16), 0.0, P(16),
                                None, None) == 4
    # total_tokens beyond batch * max_seqlen is invalid
    assert L.fp8attn_varlen_fwd(P(16), P(16), P(16), P(16), 1, 8, 9, 8, 128, P(16), 0.0, P(16),
                                None, None) == 1
    # misaligned pointers are rejected
    assert L.fp8attn_varlen_fwd(P(17), P(16), P(16), P(16), 1, 8, 8, 8, 128, P(16), 0.0, P(16),
                                None, None) == 1
    # zero tokens is a no-op
    assert L.fp8attn_varlen_fwd(None, None, None, P(16), 1, 8, 0, 8, 128, None, 0.0, None,
                                None, None) == 0
    # an unknown P rule or work schedule is invalid; the known ones pass the
    # checks (zero tokens: nothing launched)
    for rule, sched, want in ((0, 3, 1), (0, -1, 1), (2, 0, 1), (1, 2, 0), (0, 1, 0)):
        assert L.fp8attn_varlen_fwd_sched(None, None, None, P(16), 1, 8, 0, 8, 128, None, 0.0,
                                          rule, sched, None, None, None) == want
    assert L.fp8attn_create(0, P(256), 1 << 20, None, ctypes.byref(P())) == 1
    assert L.fp8attn_e4m3_encode(None, 5, 1.0, None, None) == 1
    # the amax-only entry point rejects a null context, a null output, a bad
    # head_dim and misaligned sources before any CUDA call
    f3 = P(256)
    assert L.fp8attn_amax_qkv(None, P(16), P(16), P(16), 1024, 128, None, P(16), 1, 8, 8, 8,
                              128, f3, None) == 1
    assert L.fp8attn_amax_qkv(P(64), P(16), P(16), P(16), 1024, 128, None, P(16), 1, 8, 8, 8,
                              128, None, None) == 1
    assert L.fp8attn_amax_qkv(P(64), P(16), P(16), P(16), 1024, 128, None, P(16), 1, 8, 8, 8,
                              64, f3, None) == 4
    assert L.fp8attn_amax_qkv(P(64), P(17), P(16), P(16), 1024, 128, None, P(16), 1, 8, 8, 8,
                              128, f3, None) == 4
    # the wait self-test checks its limit (0 < limit <= 1 s) and output first
    n = ctypes.c_int(0)
    assert L.fp8attn_selftest_bounded_waits(ctypes.c_uint64(0), ctypes.byref(n), None) == 1
    assert L.fp8attn_selftest_bounded_waits(ctypes.c_uint64(2 * 10**9), ctypes.byref(n), None) == 1
    assert L.fp8attn_selftest_bounded_waits(ctypes.c_uint64(10**6), None, None) == 1
    # the static cast inside attention: no context -> INVALID, before any
    # other argument is read
    assert L.fp8attn_varlen_fwd_static(None, 0, P(16), P(16), P(16), 1024, 128, P(16), 1, 8, 8,
                                       8, 128, 0.0, 0, P(16), None) == 1
    # the grouped cast: STATIC / RING only, groups dividing the heads, checked
    # before any CUDA call (mode DYNAMIC = 0, STATIC = 1, RING = 3)
    g = (P(16), P(16), P(16), 1024, 128, None, P(16), 1, 8, 8, 8, 128)
    outs = (P(16), P(16), P(16), None)
    assert L.fp8attn_quantize_qkv_grouped(P(64), 0, 0, *g, 2, *outs) == 1    # DYNAMIC
    assert L.fp8attn_quantize_qkv_grouped(P(64), 0, 2, *g, 2, *outs) == 1    # SKIP
    assert L.fp8attn_quantize_qkv_grouped(P(64), 0, 3, *g, 3, *outs) == 1    # 8 % 3
    assert L.fp8attn_quantize_qkv_grouped(P(64), 0, 3, *g, 0, *outs) == 1
    # head regrouping: sizes, groups, direction, alignment and overlap are
    # checked on the host; zero tokens is a no-op
    src, dst = P(1 << 20), P(1 << 24)
    assert L.fp8attn_regroup_heads(src, dst, -1, 8, 2, 256, 1, None) == 1
    assert L.fp8attn_regroup_heads(src, dst, 64, 8, 3, 256, 1, None) == 1    # 8 % 3
    assert L.fp8attn_regroup_heads(src, dst, 64, 8, 0, 256, 1, None) == 1
    assert L.fp8attn_regroup_heads(src, dst, 64, 8, 2, 256, 2, None) == 1    # direction
    assert L.fp8attn_regroup_heads(None, dst, 64, 8, 2, 256, 1, None) == 1
    assert L.fp8attn_regroup_heads(src, P((1 << 20) + 4096), 64, 8, 2, 256, 1, None) == 1
    assert L.fp8attn_regroup_heads(src, dst, 64, 8, 2, 100, 1, None) == 4    # 100 % 16
    assert L.fp8attn_regroup_heads(P((1 << 20) + 8), dst, 64, 8, 2, 256, 1, None) == 4
    assert L.fp8attn_regroup_heads(None, None, 0, 8, 2, 256, 0, None) == 0


def test_scale_file_round_trip(tmp_path, golden_dir):
    import quantization_amax_reduce_b200 as qar
    g = json.load(open(os.path.join(golden_dir, "static_scale_file.json")))
    p = tmp_path / "scales.json"
    p.write_text(json.dumps(g["map"]))
    m = qar.load_scale_file(str(p))
    assert m["visual.blocks.0.attn.attn"] == (224.0, 198.0, 210.0)
    assert m["visual.blocks.1.attn.attn"] == (218.0, 195.0, 207.0)
    p2 = tmp_path / "alias.json"
    p2.write_text(json.dumps(g["alias_map"]))
    assert qar.load_scale_file(str(p2))["visual.blocks.0.attn.attn"] == (224.0, 198.0, 210.0)
    out = tmp_path / "saved.json"
    qar.save_scale_file(str(out), ["a", "b"], np.array([[1.5, 3.0, 4.5], [6.0, 7.5, 9.0]]))
    assert qar.load_scale_file(str(out)) == {"a": (1.5, 3.0, 4.5), "b": (6.0, 7.5, 9.0)}


def test_scale_file_margin_on_load(tmp_path, golden_dir):
    """The alternative reading of the static values (margin applied when the
    file is read, not when it was written): each value becomes
    fl32(value * margin); the default leaves the stored values as they are."""
    import quantization_amax_reduce_b200 as qar
    g = json.load(open(os.path.join(golden_dir, "static_scale_file.json")))
    p = tmp_path / "scales.json"
    p.write_text(json.dumps(g["map"]))
    m = qar.load_scale_file(str(p), margin=1.5)
    assert m["visual.blocks.0.attn.attn"] == (336.0, 297.0, 315.0)
    p2 = tmp_path / "odd.json"
    p2.write_text(json.dumps({"x": {"q": 0.1, "k": 3.0, "v": 1e-3}}))
    got = qar.load_scale_file(str(p2), margin=1.5)["x"]
    want = tuple(float(np.float32(np.float32(v) * np.float32(1.5))) for v in (0.1, 3.0, 1e-3))
    assert got == want
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        with pytest.raises(ValueError):
            qar.load_scale_file(str(p), margin=bad)


def test_padded_source_rows_checked_on_the_host():
    """A padded source given with host-side cu_seqlens / src_seq_start is
    checked before any launch: every sequence's rows lie inside the source."""
    from quantization_amax_reduce_b200 import _check_padded_rows
    _check_padded_rows([0, 300, 301, 430], [0, 320, 640], 960)       # fits
    _check_padded_rows([0, 320, 320], [0, 960], 960)                  # empty at the end
    with pytest.raises(ValueError, match="outside"):
        _check_padded_rows([0, 300, 301, 430], [0, 320, 850], 960)    # 850 + 129 > 960
    with pytest.raises(ValueError, match="outside"):
        _check_padded_rows([0, 10], [-1], 960)
    with pytest.raises(ValueError, match="one entry"):
        _check_padded_rows([0, 10, 20], [0], 960)
    with pytest.raises(ValueError, match="decrease"):
        _check_padded_rows([0, 10, 5], [0, 320], 960)


def test_plain_c_consumer(tmp_path):
    """The C ABI is usable from C99 with nothing but include/fp8attn.h and the
    shared library: tests/c_abi/host_calls.c exercises the host-side entry
    points and argument checks (no GPU needed)."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler on this machine")
    lib_dir = os.path.join(ROOT, "quantization_amax_reduce_b200")
    exe = str(tmp_path / "host_calls")
    subprocess.check_call([cc, "-std=c99", "-Wall", "-Wextra", "-Werror",
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c_abi", "host_calls.c"),
                           "-L", lib_dir, "-lfp8attn", f"-Wl,-rpath,{lib_dir}", "-o", exe])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


def test_noalloc_sources_checked_before_any_launch(monkeypatch):
    """The allocation-free entry point runs the same host-side source checks
    as Context.quantize_qkv: a total_tokens beyond the packed source's rows
    and a padded layout whose sequences leave the source raise before the
    library is called.  (CPU tensors stand in for device ones here; the
    binding's device check is switched off and the library must not be
    reached.)"""
    import quantization_amax_reduce_b200 as qar

    def no_launch():
        raise AssertionError("the library was called")

    monkeypatch.setattr(qar, "_require_cuda", lambda t, name: None)
    monkeypatch.setattr(qar, "lib", no_launch)
    q = torch.zeros(128, 2, 128, dtype=torch.bfloat16)
    o = torch.zeros(129, 2, 128, dtype=torch.uint8)
    ds = torch.zeros(3, dtype=torch.float32)
    with pytest.raises(ValueError, match="source rows"):
        qar.quantize_qkv_noalloc(q, q, q, [0, 100, 129], 100, o, o, o, ds, total_tokens=129)
    padded = torch.zeros(2, 64, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="outside"):
        # the second sequence has 70 rows but starts at row 64 of 128
        qar.quantize_qkv_noalloc(padded, padded, padded, [0, 60, 130], 70, o, o, o, ds,
                                 total_tokens=130, src_seq_start=[0, 64])
    with pytest.raises(ValueError, match="total_tokens is required"):
        qar.quantize_qkv_noalloc(padded, padded, padded, [0, 60, 120], 64, o, o, o, ds,
                                 src_seq_start=[0, 64])
    with pytest.raises(ValueError, match="needed"):
        qar.quantize_qkv_noalloc(q, q, q, [0, 100, 128], 100, o, o, o,
                                 torch.zeros(2, dtype=torch.float32))


def test_scale_map_parsing_and_margin_in_the_library(tmp_path):
    """The scale-map reader and writer and the margin multiply are the C
    library's (fp8attn_scale_map_parse/_format, fp8attn_apply_margin): alias
    precedence, unknown keys, errors, exact fp32 round trips."""
    import quantization_amax_reduce_b200 as qar
    vals = np.array([0.1, 3.0, 1e-3, 448.0, 2.0e38, 224.0, 1.5e-40], dtype=np.float32)
    want = (vals * np.float32(1.5)).astype(np.float32)
    np.testing.assert_array_equal(qar.apply_margin(vals, 1.5), want)
    for bad in (0.0, -2.0, float("inf"), float("nan")):
        with pytest.raises(qar.FP8AttnError):
            qar.apply_margin(vals, bad)
    # the short key wins over its alias; other keys are ignored
    p = tmp_path / "m.json"
    p.write_text('{"a": {"q_scale": 9, "q": 1.25, "k": 2, "v_scale": 3.5, "note": [1, {"x": null}]},'
                 ' "b\\"c": {"q": 0.1, "k": 1e-3, "v": 7}}')
    m = qar.load_scale_file(str(p))
    assert m == {"a": (1.25, 2.0, 3.5),
                 'b"c': (float(np.float32(0.1)), float(np.float32(1e-3)), 7.0)}
    # errors: malformed text, a missing value, trailing text
    for text in ('{"a": {"q": 1, "k": 2}}', '{"a": {"q": 1, "k": 2, "v": }}', '{"a": 1}',
                 '{"a": {"q": 1, "k": 2, "v": 3}} x', '[1, 2]', '{"a": {"q": "1", "k": 2, "v": 3}}'):
        p.write_text(text)
        with pytest.raises(ValueError):
            qar.load_scale_file(str(p))
    # round trip of awkward values through the writer
    out = tmp_path / "o.json"
    names = ["visual.blocks.0.attn", 'with "quote" and \\ slash']
    arr = np.array([[0.1, 1e-3, 3.0e38], [224.0, 1.5e-40, 0.5]], dtype=np.float32)
    qar.save_scale_file(str(out), names, arr)
    back = qar.load_scale_file(str(out))
    assert list(back) == names
    for n, row in zip(names, arr):
        assert back[n] == tuple(float(x) for x in row)
    # the file is plain JSON that a generic reader accepts too
    assert set(json.load(open(out))) == set(names)
