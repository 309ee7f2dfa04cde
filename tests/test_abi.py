"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/mala.h declares, the ctypes structs match the C
layout, and invalid arguments are rejected before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from tile_skipping_causal_b200 import build, mala

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mala.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mala.load_library()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mala_[a-z_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert _declared_functions() == sorted(mala.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", mala.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (mala_\w+)", out))
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(lib, name)
    # nothing else leaks out of the library under the mala_ prefix
    assert exported == set(_declared_functions())


def test_version_and_status_strings(lib):
    assert lib.mala_version().decode().count(".") == 2
    for code, name in [(0, "MALA_OK"), (1, "MALA_ERR_INVALID_ARG"), (2, "MALA_ERR_UNSUPPORTED"),
                       (3, "MALA_ERR_WORKSPACE"), (4, "MALA_ERR_CUDA"), (5, "MALA_ERR_TIMEOUT")]:
        assert lib.mala_status_string(code).decode() == name


def _c_layout(struct, fields):
    """sizeof/offsetof of a struct in include/mala.h, from a gcc-built probe."""
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"mala.h\"\nint main(void){\n"
    prog += f'printf("%zu\\n", sizeof({struct}));\n'
    for f in fields:
        prog += f'printf("%zu\\n", offsetof({struct}, {f}));\n'
    prog += "return 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "probe.c")
        exe = os.path.join(d, "probe")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        vals = [int(x) for x in subprocess.run([exe], capture_output=True, text=True,
                                               check=True).stdout.split()]
    return vals[0], vals[1:]


@pytest.mark.parametrize("cls,name", [(mala.FwdArgs, "mala_fwd_args"),
                                      (mala.BwdArgs, "mala_bwd_args"),
                                      (mala.DecodeArgs, "mala_decode_args")])
def test_ctypes_structs_match_c_layout(cls, name):
    fields = [f[0] for f in cls._fields_]
    size, offs = _c_layout(name, fields)
    assert ctypes.sizeof(cls) == size
    assert [getattr(cls, f).offset for f in fields] == offs


def _fwd_args(**kw):
    a = mala.FwdArgs()
    fake = 0x10000
    a.q = a.k = a.v = a.o = a.lse = fake
    a.batch, a.heads_q, a.heads_kv = 1, 4, 2
    a.seqlen_q = a.seqlen_k = 256
    a.head_dim = 128
    for s in ("q_stride", "o_stride"):
        setattr(a, s, mala._i64x3(256 * 4 * 128, 4 * 128, 128))
    for s in ("k_stride", "v_stride"):
        setattr(a, s, mala._i64x3(256 * 2 * 128, 2 * 128, 128))
    a.block_q = a.block_k = 128
    a.tau = 0.1
    a.dtype = mala.MALA_BF16
    a.mode = mala.MALA_CAUSAL
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), mala.MALA_ERR_INVALID_ARG),
    (dict(lse=None), mala.MALA_ERR_INVALID_ARG),
    (dict(tau=-1.0), mala.MALA_ERR_INVALID_ARG),
    (dict(tau=float("nan")), mala.MALA_ERR_INVALID_ARG),
    (dict(heads_kv=3), mala.MALA_ERR_INVALID_ARG),
    (dict(batch=0), mala.MALA_ERR_INVALID_ARG),
    (dict(seqlen_q=0, seqlen_k=0), mala.MALA_ERR_INVALID_ARG),
    (dict(q=0x10008), mala.MALA_ERR_INVALID_ARG),           # misaligned base
    (dict(q_stride=mala._i64x3(256 * 4 * 128, 4 * 128 + 3, 128)), mala.MALA_ERR_INVALID_ARG),
    (dict(head_dim=96), mala.MALA_ERR_UNSUPPORTED),
    (dict(seqlen_k=128), mala.MALA_ERR_UNSUPPORTED),         # causal needs Nq <= Nk
    (dict(block_q=48), mala.MALA_ERR_UNSUPPORTED),
    (dict(mode=mala.MALA_DECODE), mala.MALA_ERR_UNSUPPORTED),
    (dict(dtype=7), mala.MALA_ERR_INVALID_ARG),
    (dict(wait_limit_ns=-1), mala.MALA_ERR_INVALID_ARG),
])
def test_fwd_rejects_bad_arguments_without_launching(lib, kw, code):
    a = _fwd_args(**kw)
    rc = lib.mala_fwd(ctypes.byref(a), None, 0, None)
    assert rc == code, lib.mala_last_error_message()
    assert lib.mala_last_error_message().decode()


def test_bad_head_map_rejected(lib):
    arr = (ctypes.c_int32 * 4)(0, 1, 2, 0)          # 2 is out of range for 2 KV heads
    a = _fwd_args(q_to_kv=ctypes.cast(arr, ctypes.c_void_p))
    assert lib.mala_fwd(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_INVALID_ARG


def test_null_args_rejected(lib):
    assert lib.mala_fwd(None, None, 0, None) == mala.MALA_ERR_INVALID_ARG
    assert lib.mala_bwd(None, None, 0, None) == mala.MALA_ERR_INVALID_ARG
    assert lib.mala_decode(None, None, 0, None) == mala.MALA_ERR_INVALID_ARG


def test_mask_pack_roundtrip():
    import numpy as np
    import torch
    rng = np.random.default_rng(0)
    m = rng.random((2, 3, 5, 70)) < 0.4
    w = torch.from_numpy(mala.pack_mask(m))
    assert w.shape == (2, 3, 5, 3)
    assert (mala.unpack_mask(w, 70) == m).all()


# ------------------------------------------------- packed sequences (host checks)

def _cu(*vals):
    arr = (ctypes.c_int32 * len(vals))(*vals)
    return arr, ctypes.cast(arr, ctypes.c_void_p)


@pytest.mark.parametrize("cq,ck,extra,code", [
    ((0, 100, 256), None, {}, mala.MALA_ERR_INVALID_ARG),                  # only one of the two arrays
    ((1, 100, 256), (0, 100, 256), {}, mala.MALA_ERR_INVALID_ARG),          # not starting at 0
    ((0, 100, 200), (0, 100, 256), {}, mala.MALA_ERR_INVALID_ARG),          # not ending at the total
    ((0, -1, 256), (0, 100, 256), {}, mala.MALA_ERR_INVALID_ARG),           # decreasing
    ((0, 150, 256), (0, 100, 256), {}, mala.MALA_ERR_UNSUPPORTED),          # a sequence with N_q > N_k
    ((0, 100, 256), (0, 100, 256), {"block_q": 64, "block_k": 64}, mala.MALA_ERR_UNSUPPORTED),
    ((0, 100, 256), (0, 100, 256), {"dtype": mala.MALA_FP32}, mala.MALA_ERR_UNSUPPORTED),
])
def test_packed_offsets_rejected_without_launching(lib, cq, ck, extra, code):
    keep = []
    kw = dict(batch=2, **extra)
    arr, ptr = _cu(*cq)
    keep.append(arr)
    kw["cu_seqlens_q"] = ptr
    if ck is not None:
        arr, ptr = _cu(*ck)
        keep.append(arr)
        kw["cu_seqlens_k"] = ptr
    a = _fwd_args(**kw)
    rc = lib.mala_fwd(ctypes.byref(a), None, 0, None)
    assert rc == code, lib.mala_last_error_message()
    assert lib.mala_last_error_message().decode()


def test_packed_sequence_count_limit(lib):
    n = 129                                   # one more than the packed-sequence limit
    cq = [0] + [2 * (s + 1) for s in range(n)]
    arr_q, ptr_q = _cu(*cq)
    arr_k, ptr_k = _cu(*cq)
    a = _fwd_args(batch=n, seqlen_q=cq[-1], seqlen_k=cq[-1], cu_seqlens_q=ptr_q, cu_seqlens_k=ptr_k)
    assert lib.mala_fwd(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_UNSUPPORTED
    assert "128" in lib.mala_last_error_message().decode()


def test_backward_rejects_a_negative_wait_limit(lib):
    a = mala.BwdArgs()
    fake = 0x10000
    a.q = a.k = a.v = a.o = a.dout = a.lse = a.dq = a.dk = a.dv = fake
    a.batch, a.heads_q, a.heads_kv = 2, 4, 2
    a.seqlen_q = a.seqlen_k = 256
    a.head_dim = 128
    for s in ("q_stride", "o_stride", "do_stride", "dq_stride"):
        setattr(a, s, mala._i64x3(256 * 4 * 128, 4 * 128, 128))
    for s in ("k_stride", "v_stride", "dk_stride", "dv_stride"):
        setattr(a, s, mala._i64x3(256 * 2 * 128, 2 * 128, 128))
    a.block_q = a.block_k = 128
    a.tau = 0.1
    a.dtype = mala.MALA_BF16
    a.wait_limit_ns = -1
    assert lib.mala_bwd_workspace_size(ctypes.byref(a)) == 0
    assert lib.mala_bwd(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_INVALID_ARG
    assert "wait_limit_ns" in lib.mala_last_error_message().decode()


def test_backward_checks_packed_offsets_too(lib):
    a = mala.BwdArgs()
    fake = 0x10000
    a.q = a.k = a.v = a.o = a.dout = a.lse = a.dq = a.dk = a.dv = fake
    a.batch, a.heads_q, a.heads_kv = 2, 4, 2
    a.seqlen_q = a.seqlen_k = 256
    a.head_dim = 128
    for s in ("q_stride", "o_stride", "do_stride", "dq_stride"):
        setattr(a, s, mala._i64x3(256 * 4 * 128, 4 * 128, 128))
    for s in ("k_stride", "v_stride", "dk_stride", "dv_stride"):
        setattr(a, s, mala._i64x3(256 * 2 * 128, 2 * 128, 128))
    a.block_q = a.block_k = 128
    a.tau = 0.1
    a.dtype = mala.MALA_BF16
    arr_q, a.cu_seqlens_q = _cu(0, 200, 256)
    arr_k, a.cu_seqlens_k = _cu(0, 100, 256)         # the first sequence has more queries than keys
    assert lib.mala_bwd_workspace_size(ctypes.byref(a)) == 0
    assert lib.mala_bwd(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_UNSUPPORTED


def _decode_args(**kw):
    a = mala.DecodeArgs()
    fake = 0x10000
    a.q = a.k = a.v = a.o = a.lse = fake
    a.batch, a.heads_q, a.heads_kv, a.seqlen_k, a.head_dim = 2, 8, 2, 1000, 128
    for s in ("q_stride", "o_stride"):
        setattr(a, s, mala._i64x3(8 * 128, 8 * 128, 128))
    for s in ("k_stride", "v_stride"):
        setattr(a, s, mala._i64x3(1000 * 2 * 128, 2 * 128, 128))
    a.block_k = 128
    a.tau = 0.1
    a.dtype = mala.MALA_BF16
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("kw", [dict(group_vote=2), dict(group_vote=-1), dict(kv_dtype=5),
                                dict(kv_dtype=mala.MALA_FP8_E4M3, k_scale=0.0, v_scale=1.0),
                                dict(num_splits=9), dict(wait_limit_ns=-5)])
def test_decode_rejects_bad_arguments_without_launching(lib, kw):
    a = _decode_args(**kw)
    assert lib.mala_decode_workspace_size(ctypes.byref(a)) == 0
    assert lib.mala_decode(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_INVALID_ARG
    assert lib.mala_last_error_message().decode()


@pytest.mark.parametrize("kw,code", [
    (dict(group_vote=2), mala.MALA_ERR_INVALID_ARG),
    (dict(group_vote=1, dtype=mala.MALA_FP32), mala.MALA_ERR_UNSUPPORTED),
    (dict(group_vote=1, block_q=64, block_k=64), mala.MALA_ERR_UNSUPPORTED),
    (dict(group_vote=1, heads_q=32, heads_kv=2,
          q_stride=mala._i64x3(256 * 32 * 128, 32 * 128, 128)), mala.MALA_ERR_UNSUPPORTED),   # G = 16
])
def test_fwd_group_vote_rejections(lib, kw, code):
    a = _fwd_args(**kw)
    assert lib.mala_fwd(ctypes.byref(a), None, 0, None) == code, lib.mala_last_error_message()


def test_fwd_group_vote_needs_the_default_head_map(lib):
    arr = (ctypes.c_int32 * 4)(1, 0, 0, 1)          # valid, but not h -> h / 2
    a = _fwd_args(group_vote=1, q_to_kv=ctypes.cast(arr, ctypes.c_void_p))
    assert lib.mala_fwd(ctypes.byref(a), None, 0, None) == mala.MALA_ERR_UNSUPPORTED
    assert "head map" in lib.mala_last_error_message().decode()


def test_binding_refuses_host_tensors(lib):
    """No CPU fallback: every entry point raises on host tensors."""
    import torch
    q = torch.zeros(1, 128, 4, 128, dtype=torch.bfloat16)
    k = torch.zeros(1, 128, 2, 128, dtype=torch.bfloat16)
    lse = torch.zeros(1, 4, 128)
    keep = torch.zeros(1, 4, 1, 1, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        mala.mala_fwd(q, k, k, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        mala.mala_bwd(q, k, k, q, q, lse, 0.1, keep)
    q1 = q[:, :1]
    with pytest.raises(ValueError, match="CUDA"):
        mala.mala_decode(q1, k, k, 0.1)
    with pytest.raises(ValueError, match="CUDA"):
        mala.mala_decode_noalloc(q1, k, k, 0.1, group_vote=True)


def test_c_program_links_and_runs(lib):
    """A plain C consumer: compiles against include/mala.h, links libmala.so
    and calls the host-only entry points (no GPU needed). An argument error
    comes back as a status code with a message, before anything launches."""
    prog = r'''
#include <stdio.h>
#include <string.h>
#include "mala.h"
int main(void) {
  mala_decode_args a;
  memset(&a, 0, sizeof(a));
  int rc = mala_decode(&a, NULL, 0, NULL);          /* NULL tensors: rejected on the host */
  printf("%s %s %d %s\n", mala_version(), mala_status_string(MALA_ERR_TIMEOUT), rc,
         mala_last_error_message()[0] ? "msg" : "nomsg");
  printf("%zu\n", mala_decode_workspace_size(&a));
  return rc == MALA_ERR_INVALID_ARG ? 0 : 1;
}
'''
    libdir = os.path.dirname(mala.LIB_PATH)
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "consumer.c")
        exe = os.path.join(d, "consumer")
        open(c, "w").write(prog)
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), c, "-o", exe,
                        "-L", libdir, "-lmala", "-Wl,-rpath," + libdir], check=True)
        out = subprocess.run([exe], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    first, second = out.stdout.split("\n")[:2]
    assert first.split()[1:] == ["MALA_ERR_TIMEOUT", str(mala.MALA_ERR_INVALID_ARG), "msg"]
    assert second == "0"


def test_decode_marshalling_fills_every_field(monkeypatch):
    """The binding's decode struct, filled from host tensors with the CUDA
    guard patched out (nothing is called): shapes, strides, element types,
    scales and the group-voting flag reach the C struct."""
    import torch
    monkeypatch.setattr(mala, "_require_cuda", lambda *ts: None)
    q = torch.zeros(3, 1, 8, 128, dtype=torch.bfloat16)
    k = torch.zeros(3, 1000, 2, 128, dtype=torch.float8_e4m3fn)
    o, lse, keep, a, keep_alive = mala._decode_call(q, k, k, 0.5, 128, 2, None, None, None, True, None, None,
                                                    0.25, 4.0, True)
    assert (a.batch, a.heads_q, a.heads_kv, a.seqlen_k, a.head_dim) == (3, 8, 2, 1000, 128)
    assert list(a.k_stride) == [1000 * 2 * 128, 2 * 128, 128] and list(a.q_stride) == [8 * 128, 8 * 128, 128]
    assert a.kv_dtype == mala.MALA_FP8_E4M3 and (a.k_scale, a.v_scale) == (0.25, 4.0)
    assert a.group_vote == 1 and a.num_splits == 2 and a.block_k == 128 and a.tau == 0.5
    assert a.dtype == mala.MALA_BF16
    assert a.o == o.data_ptr() and a.lse == lse.data_ptr() and a.keep_mask == keep.data_ptr()
    assert keep.shape == (3, 8, 1) and lse.shape == (3, 8)
    kb = torch.zeros(3, 1000, 2, 128, dtype=torch.bfloat16)
    _, _, keep2, a2, _ = mala._decode_call(q, kb, kb, 0.5, 128, 0, None, None, None, False, None, None,
                                           1.0, 1.0, False)
    assert a2.kv_dtype == mala.MALA_BF16 and a2.group_vote == 0 and keep2 is None and not a2.keep_mask
    with pytest.raises(ValueError):
        mala._decode_call(q, k, kb, 0.5, 128, 0, None, None, None, True, None, None, 1.0, 1.0, False)
