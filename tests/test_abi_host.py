"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

The library must build for sm_100a, load, export every function include/ssm_scan.h declares,
and reject bad arguments on the host before touching the device.
"""
import ctypes
import os
import re

import pytest

import selective_state_space_15_b200 as ssm

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "ssm_scan.h")


@pytest.fixture(scope="module")
def lib():
    ssm.build()
    return ssm.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_list():
    assert declared_functions() == sorted(ssm.EXPORTED)


def test_library_exports_every_declared_function(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_binding_struct_mirrors_the_header():
    """ScanParams lists the fields of ssm_scan_params in the header's order."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    body = re.search(r"typedef struct ssm_scan_params \{(.*?)\} ssm_scan_params;", src, flags=re.S).group(1)
    names = []
    for decl in filter(None, (d.strip() for d in body.split(";"))):
        # "type name" or "type *a, *b, *c": the declarators are the words after the type
        first, *rest = decl.split(",")
        names.append(re.findall(r"(\w+)$", first)[0])
        names += [re.sub(r"[*\s]", "", r) for r in rest]
    assert names == [f[0] for f in ssm.ScanParams._fields_]
    assert (ssm.DISC_EULER, ssm.DISC_ZOH) == (0, 1)


def test_abi_version_and_status_strings(lib):
    assert lib.ssm_abi_version() == ssm.ABI_VERSION
    for code, name in ssm._STATUS.items():
        assert lib.ssm_status_string(code).decode() == name
    assert lib.ssm_status_string(99).decode() == "SSM_ERR_UNKNOWN"


def _params(**kw):
    p = ssm.ScanParams()
    p.dtype = ssm.SSM_BF16
    p.batch, p.dim, p.dstate, p.seqlen = 1, 64, 16, 128
    fake = 0x10000  # never dereferenced: every call below fails a host check first
    p.u = p.delta = p.B = p.C = p.A = p.y = fake
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,code", [
    ("u", None, 1), ("delta", None, 1), ("B", None, 1), ("C", None, 1), ("A", None, 1), ("y", None, 1),
    ("dim", 0, 1), ("dstate", 0, 1), ("seqlen", -1, 1), ("batch", -1, 1), ("dtype", 7, 1),
    ("dstate", 24, 2), ("dstate", 512, 2), ("dstate", 200, 2),
    ("x_dim_stride", 100, 1),           # row stride shorter than the sequence
    ("bc_state_stride", 100, 1),
    ("discretization", 2, 1), ("discretization", -1, 1),   # neither Euler nor zero-order hold
    ("algorithm", 3, 1), ("algorithm", -1, 1),             # no such kernel choice
])
def test_scan_rejects_bad_arguments_on_host(lib, field, value, code):
    p = _params(**{field: value})
    assert lib.ssm_scan_fwd(ctypes.byref(p), None, 0, None) == code


def test_null_params_and_varlen_checks(lib):
    assert lib.ssm_scan_fwd(None, None, 0, None) == 1
    p = _params()
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(p), None, 4, None, 0, None) == 1   # no cu_seqlens
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(p), 0x10000, -1, None, 0, None) == 1
    p2 = _params(batch=2)
    assert lib.ssm_scan_fwd_varlen(ctypes.byref(p2), 0x10000, 4, None, 0, None) == 1  # varlen needs batch 1


def test_channel_group_host_checks(lib):
    assert lib.ssm_scan_fwd(ctypes.byref(_params(ngroups=3)), None, 0, None) == 1       # 64 channels, 3 groups
    assert lib.ssm_scan_fwd(ctypes.byref(_params(ngroups=-1)), None, 0, None) == 1
    assert lib.ssm_scan_fwd(ctypes.byref(_params(ngroups=2, bc_group_stride=-8)), None, 0, None) == 1
    # a group stride shorter than one group's [dstate][seqlen] block
    assert lib.ssm_scan_fwd(ctypes.byref(_params(ngroups=2, bc_group_stride=100)), None, 0, None) == 1
    # the decode update takes one B, C per request
    p = _params(batch=8, seqlen=1, dim=32, dstate=16, ngroups=2)
    assert lib.ssm_state_update(0x10000, 4, 0x10000, 8, ctypes.byref(p), None) == 2


def test_pool_prefill_host_checks(lib):
    p = _params(seqlen=256)
    fake = 0x10000
    f = lib.ssm_scan_fwd_varlen_pool
    assert f(None, fake, 2, fake, 4, fake, None, 0, None) == 1                     # no params
    assert f(ctypes.byref(p), None, 2, fake, 4, fake, None, 0, None) == 1          # no cu_seqlens
    assert f(ctypes.byref(p), fake, 2, None, 4, fake, None, 0, None) == 1          # no pool
    assert f(ctypes.byref(p), fake, 2, fake, 4, None, None, 0, None) == 1          # no slot ids
    assert f(ctypes.byref(p), fake, 2, fake, 0, fake, None, 0, None) == 1          # empty pool
    assert f(ctypes.byref(p), fake, -1, fake, 4, fake, None, 0, None) == 1
    ph = _params(seqlen=256)
    ph.h0 = fake
    assert f(ctypes.byref(ph), fake, 2, fake, 4, fake, None, 0, None) == 1         # the pool holds h0
    ph = _params(seqlen=256)
    ph.h_last = fake
    assert f(ctypes.byref(ph), fake, 2, fake, 4, fake, None, 0, None) == 1         # ... and h_last
    assert f(ctypes.byref(p), fake, 0, fake, 4, fake, None, 0, None) == 0          # nothing to do


def test_state_update_host_checks(lib):
    p = _params(batch=8, seqlen=1, dim=32, dstate=16)
    fake = 0x10000
    assert lib.ssm_state_update(None, 4, fake, 8, ctypes.byref(p), None) == 1
    assert lib.ssm_state_update(fake, 4, None, 8, ctypes.byref(p), None) == 1
    assert lib.ssm_state_update(fake, 0, fake, 8, ctypes.byref(p), None) == 1
    assert lib.ssm_state_update(fake, 4, fake, 7, ctypes.byref(p), None) == 1      # batch != R
    p2 = _params(batch=8, seqlen=1, dim=32, dstate=10)
    assert lib.ssm_state_update(fake, 4, fake, 8, ctypes.byref(p2), None) == 2     # not a multiple of 4
    p2 = _params(batch=8, seqlen=1, dim=32, dstate=260)
    assert lib.ssm_state_update(fake, 4, fake, 8, ctypes.byref(p2), None) == 2     # above 256
    p3 = _params(batch=8, seqlen=2, dim=32, dstate=16)
    assert lib.ssm_state_update(fake, 4, fake, 8, ctypes.byref(p3), None) == 1     # one token only
    assert lib.ssm_state_update(fake + 4, 4, fake, 8, ctypes.byref(p), None) == 1  # pool not 16-byte aligned
    p4 = _params(batch=8, seqlen=1, dim=32, dstate=16, discretization=3)
    assert lib.ssm_state_update(fake, 4, fake, 8, ctypes.byref(p4), None) == 1     # unknown discretisation


def test_algorithm_choice_on_host(lib):
    """The sequential kernel takes dstate 16 and 32 with the Euler input matrix and 16-byte
    aligned rows; other requests for it are refused before anything runs.  Its workspace is the
    16-byte unit ticket; AUTO takes the chunked kernel."""
    seq, chunked = ssm.ALGO_SEQUENTIAL, ssm.ALGO_CHUNKED
    f = lib.ssm_scan_fwd
    assert f(ctypes.byref(_params(dstate=64, algorithm=seq)), None, 0, None) == 2
    assert f(ctypes.byref(_params(discretization=ssm.DISC_ZOH, algorithm=seq)), None, 0, None) == 2
    assert f(ctypes.byref(_params(x_dim_stride=129, seqlen=128, algorithm=seq)), None, 0, None) == 2  # odd rows
    assert f(ctypes.byref(_params(algorithm=seq)), None, 0, None) == 6          # needs its ticket
    size = lib.ssm_scan_workspace_size
    assert size(ctypes.byref(_params(algorithm=seq)), 0) == 16
    assert size(ctypes.byref(_params(dstate=32, algorithm=seq)), 0) == 16
    # AUTO takes the chunked kernel: persistent fixed-length units (ticket, flags, carries) and,
    # for packed sequences, one CTA per sequence and tile (no workspace)
    assert size(ctypes.byref(_params(batch=16, dim=1024)), 0) > 16
    assert size(ctypes.byref(_params(batch=16, dim=1024, algorithm=chunked)), 0) > 16
    assert size(ctypes.byref(_params(dim=2048, seqlen=4096)), 16) == 0
    assert size(ctypes.byref(_params(dim=2048, seqlen=4096, algorithm=seq)), 16) == 16


def test_backward_host_checks(lib):
    """ssm_scan_bwd refuses bad or unsupported requests on the host, before anything runs."""
    fake = 0x10000
    g = ssm.ScanGrads()
    for name in ("dy", "du", "ddelta", "dz", "dB", "dC", "dA"):
        setattr(g, name, fake)
    f = lib.ssm_scan_bwd
    p = _params()
    assert f(ctypes.byref(p), None, None, 0, None) == 1                              # no gradients
    g_missing = ssm.ScanGrads()
    g_missing.dy = fake
    assert f(ctypes.byref(p), ctypes.byref(g_missing), None, 0, None) == 1         # outputs missing
    pz = _params()
    pz.z = fake
    g_noz = ssm.ScanGrads()
    for name in ("dy", "du", "ddelta", "dB", "dC", "dA"):
        setattr(g_noz, name, fake)
    assert f(ctypes.byref(pz), ctypes.byref(g_noz), None, 0, None) == 1            # z given, no dz
    assert f(ctypes.byref(_params(dstate=32)), ctypes.byref(g), None, 0, None) == 2
    assert f(ctypes.byref(_params(discretization=ssm.DISC_ZOH)), ctypes.byref(g), None, 0, None) == 6  # supported
    assert f(ctypes.byref(_params(dim=64, ngroups=2)), ctypes.byref(g), None, 0, None) == 2
    assert f(ctypes.byref(_params(x_dim_stride=130, seqlen=128)), ctypes.byref(g), None, 0, None) == 2
    assert f(ctypes.byref(p), ctypes.byref(g), None, 0, None) == 6                  # SSM_ERR_WORKSPACE
    # workspace: the block checkpoints and block Delta sums (every 8 steps), and per segment its
    # Delta sum and two state arrays; 128 steps of one sequence make a single segment
    need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(p))
    ckpt, cumd = 1 * (128 // 8) * 64 * 16 * 4, 1 * (128 // 8) * 64 * 4
    seg = 1 * 1 * 64 * 4 + 2 * (1 * 1 * 64 * 16 * 4)
    assert ckpt + cumd + seg <= need <= ckpt + cumd + seg + 5 * 256
    # a long sequence is cut into segments: the per-segment arrays grow with their number
    long_need = lib.ssm_scan_bwd_workspace_size(ctypes.byref(_params(seqlen=1 << 16)))
    long_blocks = (1 << 16) // 8 * 64 * (16 + 1) * 4
    assert long_need > long_blocks + seg
    assert lib.ssm_scan_bwd_workspace_size(ctypes.byref(_params(dstate=32))) == 0


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    """ssm_scan_fwd_noalloc refuses, on the host and before anything runs, a problem whose
    scratch need exceeds SSM_NOALLOC_SCRATCH_BYTES (here the chunked kernel's hand-off carries
    of 2048 chains, 4.2 MB)."""
    p = _params(batch=64, dim=1024, seqlen=4096, algorithm=ssm.ALGO_CHUNKED)
    assert lib.ssm_scan_workspace_size(ctypes.byref(p), 0) > ssm.NOALLOC_SCRATCH_BYTES
    assert lib.ssm_scan_fwd_noalloc(ctypes.byref(p), None) == 6                  # SSM_ERR_WORKSPACE


def test_workspace_size_query_is_host_only(lib):
    p = _params()
    assert lib.ssm_scan_workspace_size(ctypes.byref(p), 0) >= 0


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(FileNotFoundError):
        ssm.load(str(tmp_path / "nope.so"))


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    """bench.kernel_source_hash: comment edits keep the committed ncu counters, code edits void them."""
    import shutil
    import sys
    root = os.path.dirname(os.path.dirname(__file__))
    sys.path.insert(0, root)
    import bench
    csrc = os.path.join(root, "selective_state_space_15_b200", "csrc")
    fake = tmp_path / "selective_state_space_15_b200" / "csrc"
    fake.mkdir(parents=True)
    for name in os.listdir(csrc):
        shutil.copy(os.path.join(csrc, name), fake / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    base = bench.kernel_source_hash()
    src = fake / "chunk_scan.cuh"
    text = src.read_text()
    src.write_text("// a new comment line\n" + text.replace("namespace ssm {", "namespace ssm {  /* note */", 1))
    assert bench.kernel_source_hash() == base
    src.write_text(text.replace("static constexpr int kNP = N + 1;", "static constexpr int kNP = N + 2;"))
    assert bench.kernel_source_hash() != base
    src.write_text(text)
    api = fake / "ssm_api.cu"
    api_text = api.read_text()
    api.write_text(api_text.replace("template <> struct Shape<16, false> { static constexpr int KI = 16,",
                                    "template <> struct Shape<16, false> { static constexpr int KI = 8,", 1))
    assert bench.kernel_source_hash() != base                      # the tile of the timed kernel
    api.write_text(api_text)
    (fake / "state_update.cuh").write_text("// decode kernel changed\nint x;\n")
    (fake / "seq_scan.cuh").write_text("// sequential kernel changed\nint y;\n")
    assert bench.kernel_source_hash() == base


def test_product_path_never_touches_the_oracle():
    """The library, its binding and its header name no oracle module, file or symbol, and the
    oracle names nothing of the library: the two share no code."""
    root = os.path.dirname(os.path.dirname(__file__))
    pkg = os.path.join(root, "selective_state_space_15_b200")
    product = [os.path.join(pkg, f) for f in os.listdir(pkg) if f.endswith(".py")]
    product += [os.path.join(pkg, "csrc", f) for f in os.listdir(os.path.join(pkg, "csrc"))]
    product += [HEADER]
    for path in product:
        text = open(path, encoding="utf-8").read()
        assert not re.search(r"\boracle\b", text), path
    for name in sorted(f for f in os.listdir(os.path.join(root, "oracle")) if f.endswith((".c", ".py"))):
        text = open(os.path.join(root, "oracle", name), encoding="utf-8").read()
        assert "selective_state_space_15_b200" not in text and "ssm_scan.h" not in text, name
        assert not re.search(r"\bcsrc\b|chunk_scan|state_update\.cuh", text), name
