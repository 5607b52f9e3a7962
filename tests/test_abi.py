"""Host-side tests of the C ABI: the library builds, loads without a GPU, exports every
entry point include/ra.h declares, and rejects bad arguments before launching anything
(no compute call is made here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from sequence_parallelism_attn_b200 import build, ra
    build.build()
    return ra.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "ra.h")).read()
    return sorted(set(re.findall(r"RA_API\s+[\w\s\*]+?\b(ra_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("ra_ring_attn_fwd", "ra_lse_merge", "ra_ulysses_seq2head",
                     "ra_ulysses_head2seq", "ra_sync_status", "ra_last_error"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    from sequence_parallelism_attn_b200 import ra
    assert sorted(ra.EXPORTED) == declared_symbols()


def test_only_ra_symbols_are_exported(lib):
    import subprocess
    from sequence_parallelism_attn_b200 import ra
    out = subprocess.run(["nm", "-D", "--defined-only", ra.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    names = sorted(l.split()[-1] for l in out.splitlines() if l.strip())
    assert names == declared_symbols()


def test_version(lib):
    from sequence_parallelism_attn_b200 import ra
    assert "sm_100a" in ra.version()


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def _attn(lib, **kw):
    a = dict(q=FAKE, k=[FAKE], v=[FAKE], P=1, B=1, H_q=2, H_kv=1, Lc=128, D=128,
             qb=None, kvb=None, scale=0.1, causal=1, ind=0, outd=1, out=FAKE, lse=FAKE)
    a.update(kw)
    P = a["P"]
    arr = ctypes.c_void_p * max(P, 1)
    ks = arr(*(a["k"] * P)[:P]) if P > 0 else None
    vs = arr(*(a["v"] * P)[:P]) if P > 0 else None
    L = max(P, 1) * a["Lc"]
    qb = a["qb"] if a["qb"] is not None else L * a["H_q"] * a["D"]
    kvb = a["kvb"] if a["kvb"] is not None else a["Lc"] * a["H_kv"] * a["D"]
    return lib.ra_ring_attn_fwd(a["q"], ks, vs, P, a["B"], a["H_q"], a["H_kv"], a["Lc"], a["D"],
                                qb, kvb, a["scale"], a["causal"], a["ind"], a["outd"], a["out"],
                                a["lse"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(P=0), 1), (dict(P=65), 1), (dict(B=0), 1), (dict(H_q=3, H_kv=2), 1),
    (dict(causal=2), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(ind=1, outd=0), 1), (dict(D=32), 2), (dict(D=96), 2), (dict(ind=1, D=48), 2),
    (dict(q=FAKE + 8), 1), (dict(q=0), 1), (dict(out=FAKE + 4), 1), (dict(lse=0), 1),
    (dict(k=[0]), 1), (dict(v=[FAKE + 2]), 1), (dict(qb=5), 1), (dict(B=2, kvb=128 * 128 + 3), 1),
    (dict(ind=5), 1),
])
def test_attention_argument_validation(lib, kw, status):
    assert _attn(lib, **kw) == status
    assert lib.ra_last_error()


def test_permute_argument_validation(lib):
    s2h, h2s = lib.ra_ulysses_seq2head, lib.ra_ulysses_head2seq
    # heads not divisible by ranks ("heads divisible by the number of GPUs")
    assert s2h(FAKE, FAKE * 2, 4, 1, 16, 6, 6, 64, 0, None) == 1
    assert b"divisible" in lib.ra_last_error()
    assert s2h(FAKE, FAKE * 2, 4, 1, 16, 3, 8, 64, 0, None) == 1   # H_out % H_in
    assert s2h(FAKE, FAKE * 2, 2, 1, 16, 2, 2, 4, 0, None) == 1    # D*2 bytes % 16
    assert s2h(FAKE + 2, FAKE * 2, 2, 1, 16, 2, 2, 64, 0, None) == 1
    assert s2h(FAKE, FAKE, 2, 1, 16, 2, 2, 64, 0, None) == 1        # aliasing
    assert s2h(FAKE, FAKE * 2, 2, 1, 0, 2, 2, 64, 0, None) == 1
    assert h2s(FAKE, FAKE * 2, 3, 1, 16, 4, 64, 0, None) == 1
    assert h2s(FAKE, FAKE * 2, 2, 1, 16, 4, 64, 7, None) == 1       # bad dtype


def test_replica_sum_argument_validation(lib):
    """ra_ulysses_replica_sum refuses bad arguments on the host, before any CUDA call."""
    f = lambda i=FAKE, o=FAKE + 4096, rows=4, H_in=8, H_out=2, D=128: (
        lib.ra_ulysses_replica_sum(i, o, rows, H_in, H_out, D, None))
    assert f(rows=0) == 1 and f(H_out=0) == 1 and f(D=0) == 1
    assert f(H_in=6, H_out=4) == 1 and b"multiple" in lib.ra_last_error()
    assert f(D=66) == 1 and b"multiple of 4" in lib.ra_last_error()
    assert f(i=FAKE + 8) == 1 and f(o=0) == 1
    assert f(o=FAKE) == 1 and b"alias" in lib.ra_last_error()


def test_scatter_argument_validation(lib):
    """The one-kernel Ulysses exchange refuses bad arguments on the host, before any CUDA
    call: the rank, the destination table (null, misaligned, aliasing the input, repeated)
    and the permute's own rules."""
    def arr(*ptrs):
        return (ctypes.c_void_p * len(ptrs))(*ptrs)
    good = arr(FAKE * 2, FAKE * 3)
    s2h = lambda i=FAKE, d=good, P=2, rank=0, B=1, Lc=16, Hi=2, Ho=4, D=64, dt=0: (
        lib.ra_ulysses_seq2head_scatter(i, d, P, rank, B, Lc, Hi, Ho, D, dt, None))
    h2s = lambda i=FAKE, d=good, P=2, rank=1, B=1, Lc=16, H=4, D=64, dt=0: (
        lib.ra_ulysses_head2seq_scatter(i, d, P, rank, B, Lc, H, D, dt, None))
    assert s2h(rank=2) == 1 and b"rank" in lib.ra_last_error()
    assert s2h(rank=-1) == 1 and h2s(rank=2) == 1
    assert s2h(d=None) == 1 and h2s(d=None) == 1
    assert s2h(d=arr(FAKE * 2, FAKE * 3 + 8)) == 1 and b"aligned" in lib.ra_last_error()
    assert s2h(d=arr(FAKE * 2, 0)) == 1
    assert s2h(d=arr(FAKE * 2, FAKE)) == 1 and b"alias" in lib.ra_last_error()
    assert h2s(d=arr(FAKE * 2, FAKE * 2)) == 1 and b"distinct" in lib.ra_last_error()
    assert s2h(Ho=6, Hi=2, P=4, d=arr(FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5)) == 1  # 6 % 4
    assert s2h(Hi=3) == 1                       # H_out % H_in
    assert s2h(D=4) == 1                        # D * 2 bytes % 16
    assert s2h(P=0) == 1 and s2h(P=65) == 1
    assert h2s(H=3) == 1 and h2s(dt=7) == 1
    assert s2h(i=FAKE + 4) == 1


def test_merge_argument_validation(lib):
    m = lib.ra_lse_merge
    assert m(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, 1, 1, 8, 6, None) == 2  # D % 4
    assert m(FAKE, FAKE * 2, FAKE, FAKE * 4, 1, 1, 8, 8, None) == 1      # o_b aliases o_a
    assert m(0, FAKE * 2, FAKE * 3, FAKE * 4, 1, 1, 8, 8, None) == 1
    assert m(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, 1, 0, 8, 8, None) == 1


def test_wait_limit_roundtrip(lib):
    old = lib.ra_set_wait_limit_ns(12345)
    assert lib.ra_set_wait_limit_ns(0) == 12345
    assert lib.ra_set_wait_limit_ns(old) == 4000000000


def test_bwd_deterministic_roundtrip(lib):
    """The process-wide switch of the backward: host state only, returns the previous value
    (any non-zero argument reads as on)."""
    old = lib.ra_set_bwd_deterministic(7)
    assert old in (0, 1)
    assert lib.ra_set_bwd_deterministic(0) == 1
    assert lib.ra_set_bwd_deterministic(old) == 0


def _bwd(lib, entry="ra_ring_attn_bwd", **kw):
    """One backward call with fake pointers (every case below fails validation first)."""
    a = dict(q=FAKE, k=[FAKE], v=[FAKE], pid=FAKE, out=FAKE, lse=FAKE, dout=FAKE, P=1, B=1,
             H_q=2, H_kv=1, Lc=128, D=128, scale=0.1, causal=1, dq=FAKE, dk=[FAKE], dv=[FAKE],
             ws=FAKE)
    a.update(kw)
    P = a["P"]
    arr = ctypes.c_void_p * max(P, 1)
    rep = lambda x: arr(*(x * max(P, 1))[:max(P, 1)])
    L = max(P, 1) * a["Lc"]
    qb, kvb = L * a["H_q"] * a["D"], a["Lc"] * a["H_kv"] * a["D"]
    if entry == "ra_ring_attn_bwd_packed":
        return lib.ra_ring_attn_bwd_packed(a["q"], rep(a["k"]), rep(a["v"]), a["pid"], a["out"],
                                           a["lse"], a["dout"], P, a["B"], a["H_q"], a["H_kv"],
                                           a["Lc"], a["D"], qb, kvb, a["scale"], a["dq"],
                                           rep(a["dk"]), rep(a["dv"]), a["ws"], None)
    return getattr(lib, entry)(a["q"], rep(a["k"]), rep(a["v"]), a["out"], a["lse"], a["dout"],
                               P, a["B"], a["H_q"], a["H_kv"], a["Lc"], a["D"], qb, kvb,
                               a["scale"], a["causal"], a["dq"], rep(a["dk"]), rep(a["dv"]),
                               a["ws"], None)


@pytest.mark.parametrize("entry", ["ra_ring_attn_bwd", "ra_ring_attn_bwd_zigzag",
                                   "ra_ring_attn_bwd_packed", "ra_ring_attn_bwd_accumulate"])
@pytest.mark.parametrize("kw,status", [
    (dict(P=0), 1), (dict(P=65), 1), (dict(H_q=3, H_kv=2), 1), (dict(scale=0.0), 1),
    (dict(D=32), 2), (dict(D=96), 2), (dict(q=FAKE + 8), 1), (dict(out=0), 1),
    (dict(lse=FAKE + 4), 1), (dict(dout=0), 1), (dict(dq=FAKE + 2), 1), (dict(ws=0), 1),
    (dict(k=[0]), 1), (dict(dk=[FAKE + 4]), 1), (dict(dv=[0]), 1),
])
def test_backward_argument_validation(lib, entry, kw, status):
    """The backward entry points refuse bad arguments on the host, before any CUDA call."""
    assert _bwd(lib, entry, **kw) == status
    assert lib.ra_last_error()


def test_backward_layout_argument_validation(lib):
    # zigzag needs an even chunk length
    assert _bwd(lib, "ra_ring_attn_bwd_zigzag", Lc=129) == 1
    assert b"even" in lib.ra_last_error()
    # packed samples need non-null, 4-byte aligned position_ids
    assert _bwd(lib, "ra_ring_attn_bwd_packed", pid=0) == 1
    assert b"position_ids" in lib.ra_last_error()
    assert _bwd(lib, "ra_ring_attn_bwd_packed", pid=FAKE + 2) == 1
    assert b"aligned" in lib.ra_last_error()
    # causal must be 0 or 1 where it is an argument
    assert _bwd(lib, "ra_ring_attn_bwd", causal=2) == 1
    assert _bwd(lib, "ra_ring_attn_bwd_zigzag", causal=-1) == 1


def test_header_is_plain_c(tmp_path):
    """include/ra.h is a C ABI: it compiles as pedantic C99 with no C++ or torch types."""
    import subprocess
    src = tmp_path / "use_header.c"
    src.write_text('#include "ra.h"\n'
                   "int main(void) { ra_status s = RA_OK; ra_dtype d = RA_BF16; (void)s; (void)d;\n"
                   "  return RA_BWD_STATIC_MAX_ROWS > 0 && RA_MAX_P > 0 ? 0 : 1; }\n")
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
                        "-I", os.path.join(ROOT, "include"), "-c", str(src), "-o",
                        str(tmp_path / "use_header.o")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_tensor_helpers_reject_bad_layouts(lib):
    """ring_attn_fwd / ring_attn_bwd refuse an unknown layout, and packed samples outside
    the causal contiguous layout, before touching a device."""
    import torch
    from sequence_parallelism_attn_b200 import ra
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    k = torch.zeros(2, 1, 4, 1, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 8)
    pid = torch.zeros(1, 8, dtype=torch.int32)
    for call in (lambda: ra.ring_attn_bwd(q, k, k, q, lse, q, True, layout="diagonal"),
                 lambda: ra.ring_attn_bwd(q, k, k, q, lse, q, True, layout="zigzag",
                                          position_ids=pid),
                 lambda: ra.ring_attn_bwd(q, k, k, q, lse, q, False, position_ids=pid),
                 lambda: ra.ring_attn_fwd(q, k, k, True, layout="diagonal"),
                 lambda: ra.ring_attn_fwd(q, k, k, False, position_ids=pid)):
        with pytest.raises(ValueError):
            call()


def _c_params():
    """name -> list of parameter kinds parsed from the RA_API declarations of ra.h."""
    text = open(os.path.join(ROOT, "include", "ra.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    out = {}
    for m in re.finditer(r"RA_API\s+[\w\s\*]+?\b(ra_\w+)\s*\(([^)]*)\)\s*;", text):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        kinds = []
        for p in params:
            p = " ".join(p.split())
            if "*" in p:
                kinds.append("ptr")
            elif p.startswith("unsigned long long"):
                kinds.append("u64")
            elif p.startswith("long long"):
                kinds.append("i64")
            elif p.startswith("float"):
                kinds.append("f32")
            elif p.startswith("int") or p.startswith("ra_dtype"):
                kinds.append("i32")
            else:
                raise AssertionError(f"unmapped parameter {p!r} of {m.group(1)}")
        out[m.group(1)] = kinds
    return out


def test_binding_argtypes_match_the_header(lib):
    """Every entry point's ctypes argtypes agree with its C parameter list in ra.h."""
    kind = {ctypes.c_void_p: "ptr", ctypes.c_int: "i32", ctypes.c_longlong: "i64",
            ctypes.c_float: "f32", ctypes.c_ulonglong: "u64"}
    params = _c_params()
    assert set(params) == set(declared_symbols())
    checked = 0
    for name, want in params.items():
        argtypes = getattr(lib, name).argtypes
        if argtypes is None:
            assert want == [], f"{name} takes arguments but has no argtypes"
            continue
        assert [kind[t] for t in argtypes] == want, name
        checked += 1
    assert checked >= 12
