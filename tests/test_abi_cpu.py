"""C-ABI library checks that need no GPU: it builds for sm_100a, loads, exports
every entry point the header declares, and rejects bad arguments synchronously
before touching the device.  (Only argument combinations that fail
validation are passed here, so nothing is ever launched.)"""
import ctypes
import os
import re

import pytest

import linear_attention_blocked_b200 as la
from linear_attention_blocked_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lightning_attn.h")
HEADER_DIR = os.path.dirname(HEADER)


@pytest.fixture(scope="module")
def L():
    _build.build()
    return la.lib()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LA_API\s+[\w\s\*]*?\b(la_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("la_prefill", "la_prefill_varlen", "la_decode_step", "la_get_device_status",
                     "la_status_string", "la_prefill_workspace_size",
                     "la_prefill_varlen_workspace_size"):
        assert required in names
    assert set(names) == set(la.EXPORTED)


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_no_link_time_driver_dependency():
    # the library reaches the driver at run time; it must load without a GPU
    out = os.popen(f"ldd {_build.LIB_PATH}").read()
    assert "libcuda.so" not in out


def test_status_strings(L):
    for code in range(6):
        assert la.status_string(code)
    assert la.status_string(99) == "unknown status"


V = ctypes.c_void_p
FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _prefill(L, B=1, N=128, H=1, d=128, block=0, q=FAKE, out=FAKE, state_in=None, state_out=None,
             ws=FAKE, ws_bytes=0, dtype=0):
    return L.la_prefill(V(q), V(FAKE), V(FAKE), B, N, H, d, block, V(state_in) if state_in else None,
                        V(out), dtype, V(state_out) if state_out else None, V(ws), ws_bytes, None)


def test_prefill_argument_errors(L):
    assert _prefill(L, d=64) == la.LA_ERR_UNSUPPORTED
    assert _prefill(L, block=96) == la.LA_ERR_UNSUPPORTED
    assert _prefill(L, block=512) == la.LA_ERR_UNSUPPORTED
    assert _prefill(L, block=-1) == la.LA_ERR_INVALID_ARGUMENT
    assert _prefill(L, H=0) == la.LA_ERR_INVALID_ARGUMENT
    assert _prefill(L, B=-1) == la.LA_ERR_INVALID_ARGUMENT
    assert _prefill(L, dtype=7) == la.LA_ERR_INVALID_ARGUMENT
    assert _prefill(L, q=0) == la.LA_ERR_INVALID_ARGUMENT             # null input
    assert _prefill(L, q=FAKE + 8) == la.LA_ERR_INVALID_ARGUMENT      # misaligned
    assert _prefill(L, out=FAKE) == la.LA_ERR_INVALID_ARGUMENT        # out overlaps q
    far = 1 << 40
    assert _prefill(L, out=far, ws=0) == la.LA_ERR_WORKSPACE          # no workspace
    need = L.la_prefill_workspace_size(1, 128, 1, 128, 0)
    assert _prefill(L, out=far, ws=2 * far, ws_bytes=need - 1) == la.LA_ERR_WORKSPACE
    assert _prefill(L, out=far, ws=2 * far + 16, ws_bytes=need) == la.LA_ERR_INVALID_ARGUMENT  # ws alignment
    # state_out partially overlapping state_in
    assert _prefill(L, out=far, state_in=3 * far, state_out=3 * far + 64) == la.LA_ERR_INVALID_ARGUMENT


def test_varlen_and_decode_argument_errors(L):
    assert L.la_prefill_varlen(V(FAKE), V(FAKE), V(FAKE), None, 1, 10, 10, 1, 128, 0, None, V(FAKE), 0,
                               None, V(FAKE), 0, None) == la.LA_ERR_INVALID_ARGUMENT  # null cu_seqlens
    assert L.la_prefill_varlen(V(FAKE), V(FAKE), V(FAKE), V(FAKE), -1, 10, 10, 1, 128, 0, None, V(FAKE),
                               0, None, V(FAKE), 0, None) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_prefill_varlen(V(FAKE), V(FAKE), V(FAKE), V(FAKE), 2, 10, 10, 1, 96, 0, None, V(FAKE),
                               0, None, V(FAKE), 0, None) == la.LA_ERR_UNSUPPORTED
    assert L.la_decode_step(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 1, 1, 64, None) == \
        la.LA_ERR_UNSUPPORTED
    assert L.la_decode_step(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, -1, 1, 128, None) == \
        la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step(None, V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 1, 1, 128, None) == \
        la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step(V(FAKE + 4), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 1, 1, 128, None) == \
        la.LA_ERR_INVALID_ARGUMENT
    # output overlapping the state
    assert L.la_decode_step(V(FAKE), V(FAKE), V(FAKE), V(1 << 40), V((1 << 40) + 256), 0, 1, 1, 128,
                            None) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 0, 1, 128, None) == la.LA_OK


def test_decay_argument_errors(L):
    """The decay entry points check their arguments like the undecayed ones,
    and a missing or misaligned decay array is an argument error."""
    far = 1 << 40

    def pd(decay=FAKE, block=0, d=128, out=far):
        return L.la_prefill_decay(V(FAKE), V(FAKE), V(FAKE), 1, 128, 1, d, block, V(decay) if decay else None,
                                  None, V(out), 0, None, V(2 * far), 1 << 30, None)
    assert pd(decay=0) == la.LA_ERR_INVALID_ARGUMENT
    assert pd(decay=FAKE + 2) == la.LA_ERR_INVALID_ARGUMENT
    assert pd(d=64) == la.LA_ERR_UNSUPPORTED
    assert pd(block=64) == la.LA_ERR_UNSUPPORTED                      # decay: block 128 only
    assert pd(block=256) == la.LA_ERR_UNSUPPORTED
    assert pd(out=FAKE) == la.LA_ERR_INVALID_ARGUMENT                 # out overlaps q
    assert L.la_prefill_varlen_decay(V(FAKE), V(FAKE), V(FAKE), V(FAKE), 1, 10, 10, 1, 128, 0, None, None,
                                     V(far), 0, None, V(2 * far), 1 << 30, None) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_prefill_varlen_decay(V(FAKE), V(FAKE), V(FAKE), None, 1, 10, 10, 1, 128, 0, V(FAKE), None,
                                     V(far), 0, None, V(2 * far), 1 << 30, None) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step_decay(V(FAKE), V(FAKE), V(FAKE), None, V(FAKE), V(FAKE), 0, 1, 1, 128, None) == \
        la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step_decay(V(FAKE), V(FAKE), V(FAKE), V(FAKE + 1), V(FAKE), V(far), 0, 1, 1, 128,
                                  None) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_decode_step_decay(V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), V(FAKE), 0, 0, 1, 128,
                                  None) == la.LA_OK


def test_workspace_sizes(L):
    small = L.la_prefill_workspace_size(1, 1024, 2, 128, 0)
    big = L.la_prefill_workspace_size(1, 32768, 64, 128, 0)
    assert 0 < small < big
    assert L.la_prefill_varlen_workspace_size(8, 1 << 18, 65536, 64, 128, 0) > big
    assert L.la_prefill_workspace_size(0, 10, 1, 128, 0) == 256


def test_segment_len_control(L):
    assert L.la_set_segment_len(100) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_set_segment_len(-128) == la.LA_ERR_INVALID_ARGUMENT
    before = L.la_prefill_workspace_size(1, 65536, 64, 128, 0)
    assert L.la_set_segment_len(128) == la.LA_OK
    assert L.la_prefill_workspace_size(1, 65536, 64, 128, 0) > before
    assert L.la_set_segment_len(0) == la.LA_OK
    assert L.la_prefill_workspace_size(1, 65536, 64, 128, 0) == before
    assert L.la_debug_inject(5) == la.LA_ERR_INVALID_ARGUMENT
    assert L.la_debug_inject(0) == la.LA_OK
    assert L.la_set_wait_limit_ns(0) == la.LA_OK


def test_binding_rejects_cpu_tensors():
    """Every entry point refuses host tensors before calling the library (no
    CPU fallback exists)."""
    import torch
    q = torch.zeros(1, 128, 1, 128, dtype=torch.bfloat16)
    s = torch.zeros(1, 1, 128, 128)
    with pytest.raises(ValueError):
        la.prefill(q, q, q)
    with pytest.raises(ValueError):
        la.kv_aggregate(q, q)
    with pytest.raises(ValueError):
        la.prefill_backward(q, q, q, q)
    with pytest.raises(ValueError):
        la.state_prefix(s[None], 1)
    with pytest.raises(ValueError):
        la.decode_step(q[:, 0], q[:, 0], q[:, 0], s)


def test_slot_and_mixed_argument_errors(L):
    """The state-pool entry points reject bad arguments before launching."""
    V = ctypes.c_void_p
    fake = V(1 << 20)       # never dereferenced: validation fails first
    bad = la.LA_ERR_INVALID_ARGUMENT
    # decode rows without a slot map
    assert L.la_decode_step_slots(fake, fake, fake, fake, 4, None, fake, 0, 2, 2, 128, None) == bad
    # a pool with no slot
    assert L.la_decode_step_slots(fake, fake, fake, fake, 0, fake, fake, 0, 2, 2, 128, None) == bad
    # unsupported head dimension
    assert L.la_decode_step_slots(fake, fake, fake, fake, 4, fake, fake, 0, 2, 2, 64, None) == la.LA_ERR_UNSUPPORTED
    # prefill sequences without a slot map or without a pool
    assert L.la_prefill_varlen_slots(fake, fake, fake, fake, None, 2, 10, 8, 2, 128, 0, fake, 4, fake, 0,
                                     fake, 1 << 30, None) == bad
    assert L.la_prefill_varlen_slots(fake, fake, fake, fake, fake, 2, 10, 8, 2, 128, 0, None, 4, fake, 0,
                                     fake, 1 << 30, None) == bad
    # mixed step: empty pool, negative counts, prefill tokens without prefill sequences
    args = lambda **kw: dict(dict(q=fake, k=fake, v=fake, cu=fake, ps=fake, n_p=1, T_p=10, maxlen=10, ds=fake,
                                  n_d=2, H=2, d=128, pool=fake, n_slots=4, out=fake, od=0, ws=fake,
                                  wsb=1 << 30, sp=None, sd=None), **kw)
    call = lambda a: L.la_mixed_step(*a.values())
    assert call(args(n_slots=0)) == bad
    assert call(args(n_d=-1)) == bad
    assert call(args(n_p=0)) == bad
    assert call(args(ds=None)) == bad
    assert call(args(pool=None)) == bad
    assert call(args(d=64)) == la.LA_ERR_UNSUPPORTED


def test_sequence_parallel_argument_errors(L):
    """la_kv_aggregate and la_state_prefix reject bad arguments before launching."""
    V = ctypes.c_void_p
    fake = V(1 << 20)
    bad = la.LA_ERR_INVALID_ARGUMENT
    ws = L.la_kv_aggregate_workspace_size(1, 32768, 64, 128)
    assert ws == 2 * 148 * 128 * 128 * 4             # two partial slots per CTA range
    assert L.la_kv_aggregate_workspace_size(2, 0, 4, 128) == 0
    assert L.la_kv_aggregate_workspace_size(1, 384, 100, 128) == 2 * 100 * 128 * 128 * 4
    assert L.la_kv_aggregate(fake, fake, 1, 100, 2, 64, fake, fake, ws, None) == la.LA_ERR_UNSUPPORTED
    assert L.la_kv_aggregate(fake, fake, -1, 100, 2, 128, fake, fake, ws, None) == bad
    assert L.la_kv_aggregate(fake, fake, 1, 100, 2, 128, None, fake, ws, None) == bad          # no output
    assert L.la_kv_aggregate(None, fake, 1, 100, 2, 128, fake, fake, ws, None) == bad          # no k
    assert L.la_kv_aggregate(fake, fake, 1, 100, 2, 128, V((1 << 20) + 8), fake, ws, None) == bad  # misaligned
    assert L.la_kv_aggregate(fake, fake, 1, 100, 2, 128, V(1 << 30), None, 0, None) == la.LA_ERR_WORKSPACE
    assert L.la_kv_aggregate(fake, fake, 1, 100, 2, 128, fake, V(1 << 30), ws, None) == bad   # output inside k
    assert L.la_kv_aggregate(fake, fake, 0, 100, 2, 128, fake, None, 0, None) == la.LA_OK    # nothing to do
    assert L.la_state_prefix(fake, 1, None, fake, 4, 64, None) == la.LA_ERR_UNSUPPORTED
    assert L.la_state_prefix(fake, -1, None, fake, 4, 128, None) == bad
    assert L.la_state_prefix(None, 2, None, fake, 4, 128, None) == bad                        # no parts
    assert L.la_state_prefix(fake, 2, None, fake, 4, 128, None) == bad                        # out inside parts
    assert L.la_state_prefix(fake, 2, None, V((1 << 30) + 4), 4, 128, None) == bad            # misaligned
    assert L.la_state_prefix(fake, 2, V((1 << 30) + 1024), V(1 << 30), 4, 128, None) == bad   # partial overlap
    assert L.la_state_prefix(fake, 2, None, fake, 0, 128, None) == la.LA_OK


def test_backward_argument_errors(L):
    """la_prefill_backward rejects bad arguments before launching."""
    V = ctypes.c_void_p
    bad = la.LA_ERR_INVALID_ARGUMENT
    base = 1 << 32
    B, N, H = 1, 100, 2
    n = B * N * H * 128 * 2                      # bytes of one bf16 tensor
    q, k, v, g = (V(base + i * n) for i in range(4))
    dq, dk, dv = (V(base + (4 + i) * n) for i in range(3))
    ws_size = L.la_prefill_backward_workspace_size(B, N, H, 128)
    assert ws_size >= L.la_prefill_workspace_size(B, N, H, 128, 0) + B * H * 128 * 128 * 4  # + S_in transposed
    ws = V(base + 64 * n)
    args = lambda **kw: dict(dict(q=q, k=k, v=v, g=g, B=B, N=N, H=H, d=128, sin=None, dsout=None, dq=dq, dk=dk,
                                  dv=dv, gd=0, dsin=None, ws=ws, wsb=ws_size, s=None), **kw)
    call = lambda a: L.la_prefill_backward(*a.values())
    assert call(args(d=64)) == la.LA_ERR_UNSUPPORTED
    assert call(args(gd=7)) == bad                               # unknown gradient dtype
    assert call(args(N=-1)) == bad
    assert call(args(g=None)) == bad                             # no dout
    assert call(args(dk=dq)) == bad                              # two gradients in one buffer
    assert call(args(dv=q)) == bad                               # a gradient over an input
    assert call(args(dq=V(base + 4 * n + 8))) == bad             # misaligned
    assert call(args(ws=None)) == la.LA_ERR_WORKSPACE
    assert call(args(wsb=ws_size - 1)) == la.LA_ERR_WORKSPACE
    assert call(args(ws=V(base + 64 * n + 16))) == bad           # workspace not 256-byte aligned
    assert call(args(ws=V(base + 5 * n))) == bad                 # workspace over a gradient
    assert call(args(B=0)) == la.LA_OK                           # nothing to do


def test_backward_varlen_argument_errors(L):
    """la_prefill_backward_varlen rejects bad arguments before launching."""
    V = ctypes.c_void_p
    bad = la.LA_ERR_INVALID_ARGUMENT
    base = 1 << 32
    nseq, T, H = 3, 500, 2
    n = T * H * 128 * 2                          # bytes of one bf16 tensor
    q, k, v, g = (V(base + i * n) for i in range(4))
    dq, dk, dv = (V(base + (4 + i) * n) for i in range(3))
    cu = V(base + 40 * n)
    ws_size = L.la_prefill_backward_varlen_workspace_size(nseq, T, 300, H, 128)
    assert ws_size >= L.la_prefill_varlen_workspace_size(nseq, T, 300, H, 128, 0) + nseq * H * 128 * 128 * 4
    ws = V(base + 64 * n)
    args = lambda **kw: dict(dict(q=q, k=k, v=v, g=g, cu=cu, nseq=nseq, T=T, maxlen=300, H=H, d=128, sin=None,
                                  dsout=None, dq=dq, dk=dk, dv=dv, gd=0, dsin=None, ws=ws, wsb=ws_size, s=None), **kw)
    call = lambda a: L.la_prefill_backward_varlen(*a.values())
    assert call(args(cu=None)) == bad                            # no cu_seqlens
    assert call(args(cu=V(base + 40 * n + 2))) == bad            # cu_seqlens misaligned
    assert call(args(d=64)) == la.LA_ERR_UNSUPPORTED
    assert call(args(gd=7)) == bad
    assert call(args(T=-1)) == bad
    assert call(args(nseq=0)) == bad                             # tokens without sequences
    assert call(args(dq=g)) == bad                               # a gradient over an input
    assert call(args(ws=None)) == la.LA_ERR_WORKSPACE
    assert call(args(wsb=ws_size - 1)) == la.LA_ERR_WORKSPACE
    assert call(args(ws=cu)) == bad                              # workspace over cu_seqlens
    assert call(args(nseq=0, T=0)) == la.LA_OK                   # nothing to do


def test_host_memory_entry_point_validates_before_any_copy():
    """prefill_from_host refuses unpinned, non-bf16 or non-contiguous host
    inputs before touching a device."""
    import torch
    q = torch.zeros(1, 16, 1, 128, dtype=torch.bfloat16)
    for bad in (q, q.float(), q[:, ::2]):
        with pytest.raises(ValueError):
            la.prefill_from_host(bad, bad, bad)


def test_host_pipeline_argument_errors(L):
    """la_prefill_from_host checks shapes, the scratch size and alignment, and
    that the host buffers are pinned, before queueing anything."""
    far = 1 << 40
    need = L.la_prefill_from_host_buffer_size(1, 256, 2, 128, 0)
    assert need > 0 and L.la_prefill_from_host_buffer_size(1, 256, 2, 64, 0) == 0
    assert L.la_prefill_from_host_buffer_size(1, 256, 2, 128, 1) > need        # fp32 output slots

    def call(B=1, N=512, H=2, d=128, chunk=256, buf=far, nbytes=None, host=FAKE):
        return L.la_prefill_from_host(V(host), V(host), V(host), B, N, H, d, chunk, None, V(host), 0, None,
                                      V(buf), need if nbytes is None else nbytes, None, None, None)
    assert call(d=64) == la.LA_ERR_UNSUPPORTED
    assert call(chunk=0) == la.LA_ERR_INVALID_ARGUMENT
    assert call(N=-1) == la.LA_ERR_INVALID_ARGUMENT
    assert call(B=0) == la.LA_OK
    assert call(nbytes=need - 1) == la.LA_ERR_WORKSPACE
    assert call(buf=far + 16) == la.LA_ERR_INVALID_ARGUMENT                  # scratch alignment
    assert call() == la.LA_ERR_INVALID_ARGUMENT                              # host buffers not pinned


def test_header_is_plain_c_and_links_from_c(tmp_path):
    """The boundary as a C user sees it: a C99 translation unit that includes
    include/lightning_attn.h, takes the address of every entry point, links
    against the built library and calls its host-only functions (status
    strings, workspace sizes); no GPU is touched."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    _build.build()
    lib_dir = os.path.dirname(la.library_path())
    cuda_inc = "/usr/local/cuda/include"
    names = declared_functions()
    src = tmp_path / "use_abi.c"
    src.write_text(
        "#include <stdio.h>\n#include \"lightning_attn.h\"\n"
        "int main(void) {\n"
        "    const void *fns[] = {" + ", ".join(f"(const void *)&{n}" for n in names) + "};\n"
        "    size_t ws = la_kv_aggregate_workspace_size(1, 32768, 64, 128);\n"
        "    printf(\"%d %s %zu\\n\", (int)(sizeof fns / sizeof fns[0]), la_status_string(LA_ERR_WORKSPACE), ws);\n"
        "    return la_prefill_workspace_size(1, 1024, 2, 128, 0) > 0 ? 0 : 1;\n"
        "}\n")
    exe = tmp_path / "use_abi"
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", HEADER_DIR, "-I", cuda_inc, str(src), "-o", str(exe),
           "-L", lib_dir, "-llightning_attn", f"-Wl,-rpath,{lib_dir}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    count, rest = run.stdout.split(" ", 1)
    assert int(count) == len(names)
    assert "workspace" in rest and rest.strip().endswith(str(2 * 148 * 128 * 128 * 4))
