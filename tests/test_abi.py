"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, the ctypes struct mirrors the C layout, and host-side argument
validation rejects bad calls before any CUDA call is made."""
import ctypes
import os
import re
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def fa():
    from block_sparse_attention_create_b200 import build
    build.build()
    from block_sparse_attention_create_b200 import _binding
    return _binding


def _gpu_visible():
    """The calls here pass fake device addresses.  One that passes every host check
    would launch a kernel on them, so it is made only where no GPU is visible: there
    it fails with FA_ERR_CUDA before any launch.  With a GPU it is skipped."""
    import torch
    return torch.cuda.is_available()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_two_operations():
    syms = declared_symbols()
    assert "fa_create_block_mask" in syms and "fa_flex_attention_fwd" in syms


def test_library_exports_every_declared_symbol(fa):
    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(fa_\w+)", out))
    for s in declared_symbols():
        assert s in exported, s
        assert hasattr(fa._lib, s)
    assert set(fa.EXPORTED) == set(declared_symbols())


def test_struct_layout_matches_c(fa):
    """Compile a C probe against include/fa.h and compare offsets with ctypes."""
    fields = [f for f, _ in fa.fa_block_mask._fields_]
    src = "#include <stdio.h>\n#include <stddef.h>\n#include \"fa.h\"\nint main(void){\n"
    src += 'printf("%zu\\n", sizeof(fa_block_mask));\n'
    for f in fields:
        src += f'printf("%zu\\n", offsetof(fa_block_mask, {f}));\n'
    src += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    assert vals[0] == ctypes.sizeof(fa.fa_block_mask)
    for f, off in zip(fields, vals[1:]):
        assert getattr(fa.fa_block_mask, f).offset == off, f


def test_enum_values_match_header(fa):
    text = open(HEADER).read()
    for name in ("FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA",
                 "FA_ERR_TIMEOUT", "FA_ERR_SCRATCH_TOO_SMALL", "FA_MASK_CAUSAL", "FA_MASK_SLIDING_WINDOW_CAUSAL",
                 "FA_MASK_DOCUMENT_CAUSAL", "FA_MASK_BITMAP", "FA_SCORE_NONE", "FA_SCORE_TANH_SOFTCAP",
                 "FA_BF16", "FA_FP16"):
        m = re.search(rf"\b{name}\s*=\s*(\d+)", text)
        assert m and int(m.group(1)) == getattr(fa, name), name


def test_status_strings(fa):
    assert fa.fa_status_string(0) == b"FA_OK"
    assert fa.fa_status_string(4) == b"FA_ERR_TIMEOUT"
    assert fa.fa_status_string(99) == b"FA_ERR_UNKNOWN"


def test_block_mask_dims(fa):
    assert fa.block_mask_dims(32768, 32768) == (256, 256)
    assert fa.block_mask_dims(129, 1) == (2, 1)
    assert fa.block_mask_dims(0, 0) == (0, 0)
    nq, nkv = ctypes.c_int32(), ctypes.c_int32()
    assert fa.fa_block_mask_dims(-1, 5, 128, ctypes.byref(nq), ctypes.byref(nkv)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_block_mask_dims(5, 5, 64, ctypes.byref(nq), ctypes.byref(nkv)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_block_mask_dims(fa.FA_MAX_LEN + 1, 5, 128, ctypes.byref(nq),
                                 ctypes.byref(nkv)) == fa.FA_ERR_INVALID_ARG


def test_create_block_mask_rejects_bad_arguments(fa):
    bm = fa.fa_block_mask()
    null = ctypes.c_void_p(0)
    # unknown kind, bad window, missing doc ids, NULL struct, NULL arrays
    assert fa.fa_create_block_mask(7, 0, null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask(1, 0, null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask(2, 0, null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask(0, 0, null, 256, 256, 128, None, null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask(0, 0, null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask(0, 0, null, 256, 256, 100, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    # an empty mask is valid and launches nothing
    assert fa.fa_create_block_mask(0, 0, null, 0, 0, 128, ctypes.byref(bm), null) == fa.FA_OK
    assert (bm.q_len, bm.n_q_blocks, bm.block) == (0, 0, 128)


def test_bitmap_builder_and_transpose_reject_bad_arguments(fa):
    bm = fa.fa_block_mask()
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)            # never dereferenced: rejected first
    # NULL or misaligned bitmap, NULL struct, NULL tables, bad block
    assert fa.fa_create_block_mask_bitmap(null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask_bitmap(ctypes.c_void_p((1 << 20) + 4), 256, 256, 128,
                                          ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask_bitmap(fake, 256, 256, 128, None, null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask_bitmap(fake, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_create_block_mask_bitmap(fake, 256, 256, 64, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    # the create_block_mask entry point itself does not take the bitmap kind
    assert fa.fa_create_block_mask(3, 0, null, 256, 256, 128, ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    # empty: valid, nothing launched
    assert fa.fa_create_block_mask_bitmap(null, 0, 0, 128, ctypes.byref(bm), null) == fa.FA_OK
    assert bm.kind == fa.FA_MASK_BITMAP
    # transpose: NULL struct / outputs; an empty mask launches nothing
    assert fa.fa_block_mask_transpose(None, fake, fake, fake, fake, null) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_block_mask_transpose(ctypes.byref(bm), null, null, null, null, null) == fa.FA_OK
    bm2 = fa.fa_block_mask()
    bm2.block, bm2.n_q_blocks, bm2.n_kv_blocks = 128, 2, 2
    assert fa.fa_block_mask_transpose(ctypes.byref(bm2), fake, fake, fake, fake, null) == fa.FA_ERR_INVALID_ARG


def test_gqa_rejects_uneven_head_groups(fa):
    bm = fa.fa_block_mask()
    bm.block, bm.q_len, bm.kv_len = 128, 256, 256
    p = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any use
    null = ctypes.c_void_p(0)
    for h, hkv in ((6, 4), (4, 0), (4, -1), (2, 4)):
        assert fa.fa_flex_attention_fwd_gqa(p, p, p, 0, 1, h, hkv, 256, 256, 64, ctypes.byref(bm), 0,
                                            0.0, 0.0, p, null, p, null) == fa.FA_ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(fa):
    p = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected before any use
    null = ctypes.c_void_p(0)
    need = fa.fa_decode_workspace_bytes(1, 8, 2, 1, 1000, 64)
    assert need > 256

    def call(**kw):
        a = dict(B=1, H=8, Hkv=2, L=1, S=1000, D=64, mask=1, window=0, ws=need)
        a.update(kw)
        return fa.fa_flex_attention_decode(p, p, p, 0, a["B"], a["H"], a["Hkv"], a["L"], a["S"],
                                           a["D"], a["mask"], a["window"], 0, 0.0, 0.0, p, null, p,
                                           a["ws"], null)
    assert call(Hkv=3) == fa.FA_ERR_INVALID_ARG            # H not a multiple of Hkv
    assert call(mask=7) == fa.FA_ERR_INVALID_ARG
    assert call(mask=2, window=0) == fa.FA_ERR_INVALID_ARG
    assert call(D=96) == fa.FA_ERR_UNSUPPORTED
    assert call(H=8, Hkv=1, L=5) == fa.FA_ERR_UNSUPPORTED  # 40 rows share one K/V head
    assert call(ws=need - 4) == fa.FA_ERR_INVALID_ARG
    assert call(B=0) == fa.FA_OK                            # empty: nothing launched


def test_bh_builder_rejects_bad_arguments(fa):
    bm = fa.fa_block_mask()
    null = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected first
    for kind, mb, mh, doc, bits in ((0, 0, 1, null, null), (0, 1, -2, null, null),
                                    (2, 2, 1, null, null), (3, 1, 2, null, null), (9, 1, 1, null, null)):
        assert fa.fa_create_block_mask_bh(kind, 0, doc, bits, mb, mh, 256, 256, 128,
                                          ctypes.byref(bm), null) == fa.FA_ERR_INVALID_ARG
    # NULL tables for a non-empty mask
    assert fa.fa_create_block_mask_bh(0, 0, null, null, 2, 2, 256, 256, 128, ctypes.byref(bm),
                                      null) == fa.FA_ERR_INVALID_ARG
    # empty: valid, nothing launched, instance counts recorded
    assert fa.fa_create_block_mask_bh(3, 0, null, fake, 2, 3, 0, 0, 128, ctypes.byref(bm),
                                      null) == fa.FA_OK
    assert (bm.mask_batch, bm.mask_heads) == (2, 3)


def _fwd(fa, bm, **kw):
    args = dict(q=1024, k=1024, v=1024, dtype=0, B=1, H=1, L=256, S=256, D=64, sk=0, cap=0.0,
                scale=0.0, out=1024, lse=0, ws=1024)
    args.update(kw)
    vp = ctypes.c_void_p
    return fa.fa_flex_attention_fwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), args["dtype"],
                                    args["B"], args["H"], args["L"], args["S"], args["D"],
                                    ctypes.byref(bm) if bm is not None else None, args["sk"],
                                    args["cap"], args["scale"], vp(args["out"]), vp(args["lse"]),
                                    vp(args["ws"]), vp(0))


def test_fwd_rejects_bad_arguments_on_host(fa):
    """Every case below is refused before any CUDA call (the pointers are fake)."""
    bm = fa.fa_block_mask()
    bm.q_len, bm.kv_len, bm.block, bm.n_q_blocks, bm.n_kv_blocks = 256, 256, 128, 2, 2
    bm.kv_num_blocks = bm.full_kv_num_blocks = bm.q_order = 4096
    E = fa.FA_ERR_INVALID_ARG
    assert _fwd(fa, None) == E
    assert _fwd(fa, bm, ws=0) == E
    assert _fwd(fa, bm, dtype=5) == E
    assert _fwd(fa, bm, L=128) == E                 # L != mask q_len
    assert _fwd(fa, bm, S=512) == E                 # S != mask kv_len
    assert _fwd(fa, bm, sk=1, cap=0.0) == E         # softcap needs c > 0
    assert _fwd(fa, bm, sk=1, cap=float("inf")) == E
    assert _fwd(fa, bm, sk=3) == E
    assert _fwd(fa, bm, scale=float("nan")) == E
    assert _fwd(fa, bm, B=-1) == E
    assert _fwd(fa, bm, D=96) == fa.FA_ERR_UNSUPPORTED
    assert _fwd(fa, bm, q=1030) == E                # not 16-byte aligned
    assert _fwd(fa, bm, out=0) == E
    assert _fwd(fa, bm, k=0) == E
    # B*H == 0 or L == 0: nothing to do
    assert _fwd(fa, bm, B=0) == fa.FA_OK
    bm0 = fa.fa_block_mask()
    bm0.q_len, bm0.kv_len, bm0.block = 0, 256, 128
    assert _fwd(fa, bm0, L=0) == fa.FA_OK


def _bwd(fa, bm, **kw):
    args = dict(q=1024, k=1024, v=1024, out=1024, dout=1024, lse=1024, dtype=0, B=1, H=2, Hkv=1,
                L=256, S=256, D=64, cols=4096, sk=0, cap=0.0, scale=0.0, dq=1024, dk=1024,
                dv=1024, ws=1024, ws_bytes=None)
    args.update(kw)
    if args["ws_bytes"] is None:
        args["ws_bytes"] = fa.fa_bwd_workspace_bytes(args["B"], args["H"], args["L"])
    vp = ctypes.c_void_p
    c = vp(args["cols"])
    return fa.fa_flex_attention_bwd(vp(args["q"]), vp(args["k"]), vp(args["v"]), vp(args["out"]),
                                    vp(args["dout"]), vp(args["lse"]), args["dtype"], args["B"],
                                    args["H"], args["Hkv"], args["L"], args["S"], args["D"],
                                    ctypes.byref(bm) if bm is not None else None, c, c, c, c,
                                    args["sk"], args["cap"], args["scale"], vp(args["dq"]),
                                    vp(args["dk"]), vp(args["dv"]), vp(args["ws"]),
                                    args["ws_bytes"], vp(0))


def test_bwd_rejects_bad_arguments_on_host(fa):
    """Every case below is refused before any CUDA call (the pointers are fake)."""
    bm = fa.fa_block_mask()
    bm.q_len, bm.kv_len, bm.block, bm.n_q_blocks, bm.n_kv_blocks = 256, 256, 128, 2, 2
    bm.kv_num_blocks = bm.full_kv_num_blocks = bm.q_order = 4096
    bm.kv_indices = bm.full_kv_indices = 4096
    E, U = fa.FA_ERR_INVALID_ARG, fa.FA_ERR_UNSUPPORTED
    assert fa.fa_bwd_workspace_bytes(1, 2, 256) >= 2 * 256 * 4
    assert _bwd(fa, None) == E
    assert _bwd(fa, bm, dtype=5) == E
    assert _bwd(fa, bm, Hkv=3) == E                 # H not a multiple of H_kv
    assert _bwd(fa, bm, Hkv=0) == E
    assert _bwd(fa, bm, L=128) == E                 # L != mask q_len
    assert _bwd(fa, bm, S=512) == E                 # S != mask kv_len
    assert _bwd(fa, bm, sk=1, cap=0.0) == E
    assert _bwd(fa, bm, sk=2) == E
    assert _bwd(fa, bm, scale=float("inf")) == E
    assert _bwd(fa, bm, D=32) == U
    assert _bwd(fa, bm, ws=0) == E
    assert _bwd(fa, bm, ws_bytes=16) == E           # below fa_bwd_workspace_bytes
    assert _bwd(fa, bm, dq=0) == E
    assert _bwd(fa, bm, dv=0) == E
    assert _bwd(fa, bm, cols=0) == E                # column lists missing
    assert _bwd(fa, bm, dout=1026) == E             # not 4-byte aligned
    assert _bwd(fa, bm, out=1032) == E              # 8- but not 16-byte aligned (16-byte loads)
    assert _bwd(fa, bm, q=1028) == E                # 4- but not 16-byte aligned (cp.async source)
    assert _bwd(fa, bm, k=1032) == E
    assert _bwd(fa, bm, lse=1026) == E
    assert _bwd(fa, bm, dq=1032) == E               # gradients are written in 16-byte pieces
    assert _bwd(fa, bm, dk=1028) == E
    assert _bwd(fa, bm, dv=1040 + 4) == E
    assert _bwd(fa, bm, ws=1032) == E               # error word + row sums: 16 bytes
    assert _bwd(fa, bm, cols=4098) == E             # column lists not 4-byte aligned
    bm_doc = fa.fa_block_mask()
    ctypes.pointer(bm_doc)[0] = bm
    bm_doc.kind = fa.FA_MASK_DOCUMENT_CAUSAL        # document ids missing
    assert _bwd(fa, bm_doc) == E
    bm_bh = fa.fa_block_mask()
    ctypes.pointer(bm_bh)[0] = bm
    bm_bh.mask_heads = 3                            # per-head tables for 2 heads
    assert _bwd(fa, bm_bh) == E
    bm_bh.mask_heads = 2                            # per-(b, h) tables: past the checks
    if not _gpu_visible():
        assert _bwd(fa, bm_bh) == fa.FA_ERR_CUDA    # (no GPU here)
    # nothing to do: no query rows and no key rows
    assert _bwd(fa, bm, B=0) == fa.FA_OK


def test_workspace_size(fa):
    assert fa.fa_fwd_workspace_bytes() >= 4


def test_missing_library_fails_loudly(tmp_path):
    """With libfa.so absent the binding raises instead of falling back."""
    import shutil
    pkg = os.path.join(ROOT, "block_sparse_attention_create_b200")
    dst = tmp_path / "block_sparse_attention_create_b200"
    shutil.copytree(pkg, dst, ignore=shutil.ignore_patterns("*.so", "_build", "__pycache__"))
    code = ("import sys; sys.path.insert(0, %r); import block_sparse_attention_create_b200 as fa\n"
            "try:\n    fa.flex_attention\nexcept ImportError as e:\n    print('raised', e)\n"
            % str(tmp_path))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True)
    assert "raised" in out.stdout and "libfa.so is missing" in out.stdout, out.stdout + out.stderr


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "block_sparse_attention_create_b200")
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b)", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                assert not pat.search(open(os.path.join(dirpath, f)).read()), f


def test_ops_refuse_host_tensors(fa):
    """The torch-facing calls take device tensors only: host tensors are refused
    before the library is called (no host computation path exists)."""
    import torch
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 2, 128, dtype=torch.float32)
    with pytest.raises(ValueError):
        fa.flex_attention(q, q, q, None)
    with pytest.raises(ValueError):
        fa.flex_attention_noalloc(q, q, q, fa.FA_MASK_CAUSAL)
    with pytest.raises(ValueError):
        fa.flex_attention_decode(q, q, q)
    with pytest.raises(ValueError):
        fa.flex_attention_backward(q, q, q, q, q, lse, None)
    with pytest.raises(ValueError):
        fa.flex_attention(q.float(), q.float(), q.float(), None)   # fp32 inputs


def test_noalloc_binding_checks_shapes_before_the_call(fa):
    """flex_attention_noalloc refuses mismatched K / V, a short or missing document
    id tensor and wrongly shaped outputs, each with its own error, before anything
    reaches the library (shape checks come before the device checks, so they run
    here without a GPU)."""
    import torch
    q = torch.zeros(1, 2, 128, 64, dtype=torch.bfloat16)
    k = torch.zeros(1, 2, 256, 64, dtype=torch.bfloat16)
    cases = [
        ((q, k[:, :1], k[:, :1], fa.FA_MASK_CAUSAL), {}, "k and v"),           # fewer heads
        ((q, k[..., :32], k[..., :32], fa.FA_MASK_CAUSAL), {}, "k and v"),     # smaller D
        ((q, k, k[:, :, :128], fa.FA_MASK_CAUSAL), {}, "k and v"),             # v shorter
        ((q, k, k, fa.FA_MASK_DOCUMENT_CAUSAL), {}, "doc_id"),                  # no ids
        ((q, k, k, fa.FA_MASK_DOCUMENT_CAUSAL),
         {"doc_id": torch.zeros(200, dtype=torch.int32)}, "doc_id"),           # short ids
        ((q, k, k, fa.FA_MASK_DOCUMENT_CAUSAL),
         {"doc_id": torch.zeros(256, dtype=torch.int64)}, "doc_id"),           # wrong dtype
        ((q, k, k, fa.FA_MASK_CAUSAL), {"lse": torch.zeros(1, 2, 64)}, "lse"),  # wrong shape
        ((q, k, k, fa.FA_MASK_CAUSAL), {"lse": torch.zeros(1, 2, 128, dtype=torch.float64)}, "lse"),
        ((q, k, k, fa.FA_MASK_CAUSAL), {"out": torch.zeros(1, 2, 128, 32, dtype=torch.bfloat16)},
         "out"),
        ((q, k, k, fa.FA_MASK_CAUSAL), {"device_error": torch.zeros(1, dtype=torch.int64)},
         "device_error"),
        ((q, k, k, fa.FA_MASK_CAUSAL), {}, "CUDA"),                             # host tensors
    ]
    for args, kw, what in cases:
        with pytest.raises(ValueError, match=what):
            fa.flex_attention_noalloc(*args, **kw)


def _fake_mask(fa, nq=2, nkv=2, L=256, S=256, kind=0, base=0x10000000):
    """A block-mask struct whose device pointers are never dereferenced on the host
    (the calls below return on their argument checks before any CUDA call)."""
    bm = fa.fa_block_mask()
    bm.kv_num_blocks = base
    bm.kv_indices = base + 0x1000
    bm.full_kv_num_blocks = base + 0x2000
    bm.full_kv_indices = base + 0x3000
    bm.q_order = base + 0x4000
    bm.q_len, bm.kv_len, bm.block, bm.n_q_blocks, bm.n_kv_blocks = L, S, 128, nq, nkv
    bm.kind, bm.window = kind, 0
    bm.doc_id = base + 0x5000 if kind == 2 else None
    bm.bitmap = base + 0x6000 if kind == 3 else None
    bm.mask_batch = bm.mask_heads = 1
    return bm


def test_forward_rejects_each_misaligned_pointer_before_any_launch(fa):
    """Every pointer the forward kernel reads or writes is checked on the host:
    Q, K, V, out 16 bytes; the schedule and a bitmap 8; block lists, document ids,
    LSE and the workspace 4.  A misaligned one returns FA_ERR_INVALID_ARG; with
    every pointer aligned the call gets past the checks (to a CUDA error here,
    where there is no GPU)."""
    A = 0x20000000
    good = dict(q=A, k=A + 0x100000, v=A + 0x200000, out=A + 0x300000, lse=A + 0x400000,
                ws=A + 0x500000)
    vp = ctypes.c_void_p

    def call(ptrs, bm):
        return fa.fa_flex_attention_fwd(vp(ptrs["q"]), vp(ptrs["k"]), vp(ptrs["v"]), fa.FA_BF16,
                                        1, 2, 256, 256, 64, ctypes.byref(bm), 0, 0.0, 0.0,
                                        vp(ptrs["out"]), vp(ptrs["lse"]), vp(ptrs["ws"]), None)
    if not _gpu_visible():
        for kind in (0, 2, 3):
            assert call(good, _fake_mask(fa, kind=kind)) == fa.FA_ERR_CUDA
    for name, off in (("q", 8), ("k", 4), ("v", 2), ("out", 8), ("lse", 2), ("ws", 1)):
        bad = dict(good)
        bad[name] += off
        assert call(bad, _fake_mask(fa)) == fa.FA_ERR_INVALID_ARG, name
    for field, off, kind in (("q_order", 4, 0), ("kv_indices", 2, 0), ("full_kv_indices", 1, 0),
                             ("doc_id", 2, 2), ("bitmap", 4, 3)):
        bm = _fake_mask(fa, kind=kind)
        setattr(bm, field, getattr(bm, field) + off)
        assert call(good, bm) == fa.FA_ERR_INVALID_ARG, field


def test_decode_rejects_misaligned_pointers_before_any_launch(fa):
    vp = ctypes.c_void_p
    A = 0x20000000
    need = int(fa.fa_decode_workspace_bytes(1, 4, 1, 1, 1024, 64))
    good = dict(q=A, k=A + 0x100000, v=A + 0x200000, out=A + 0x300000, lse=A + 0x400000,
                ws=A + 0x500000)

    def call(p):
        return fa.fa_flex_attention_decode(vp(p["q"]), vp(p["k"]), vp(p["v"]), fa.FA_BF16, 1, 4, 1,
                                           1, 1024, 64, fa.FA_DECODE_CAUSAL, 0, 0, 0.0, 0.0,
                                           vp(p["out"]), vp(p["lse"]), vp(p["ws"]), need, None)
    if not _gpu_visible():
        assert call(good) == fa.FA_ERR_CUDA
    for name, off in (("q", 8), ("k", 4), ("v", 2), ("out", 8), ("lse", 2), ("ws", 8)):
        bad = dict(good)
        bad[name] += off
        assert call(bad) == fa.FA_ERR_INVALID_ARG, name
