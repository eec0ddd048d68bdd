"""The C-ABI library loads and exports every symbol include/qsa.h declares, and
its host-side validation answers without a GPU (no compute calls here)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qsa_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_long_02_b200 import build

    build.build()
    import block_sparse_long_02_b200 as m

    return m


def test_every_declared_symbol_is_exported(qsa):
    names = _declared()
    assert "qsa_decode_step" in names and len(names) >= 8
    lib = ctypes.CDLL(qsa.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(qsa.EXPORTS) <= set(names)


def test_workspace_sizes_and_config_validation(qsa):
    cfg = qsa.Config()
    n = qsa.qsa_workspace_size(cfg, qsa.OP_DECODE_STEP, 8, 262144 + 64)
    assert n >= 8 * 65536 * 4  # at least the fp32 score row per sequence
    # The step kernel's partial states (16 splits x (G x 128 + 2 G) floats per
    # sequence and kv head) and listed blocks (4096 x 8 bytes per sequence) are in it.
    assert n >= 8 * 65536 * 4 + 8 * 4 * 16 * (8 * 128 + 16) * 4 + 8 * 4096 * 8
    # The documented no-allocation limits: 8 x 256K fits the 16 MiB scratch, 64 x 4M does not.
    assert n <= 16 << 20
    assert qsa.qsa_workspace_size(cfg, qsa.OP_DECODE_STEP, 64, 4 << 20) > 16 << 20
    assert qsa.qsa_workspace_size(cfg, qsa.OP_DECODE_STEP, 16, 262144 + 64) > n  # grows with the batch
    assert qsa.qsa_workspace_size(cfg, qsa.OP_SPARSE_ATTENTION, 1, 1024, 1024) == 256
    for bad, status in ((dict(idx_heads=8), 2), (dict(head_dim=64), 2), (dict(q_heads=30, kv_heads=4), 2),
                        (dict(r=0), 2), (dict(K=0), 1), (dict(rope_dims=60), 2), (dict(kv_heads=3, q_heads=24), 2)):
        c = qsa.Config(**bad)
        with pytest.raises(qsa.QSAError) as e:
            qsa.qsa_workspace_size(c, qsa.OP_TOPK_BLOCKS, 1, 1024, 16)
        assert e.value.status == status, bad


def test_null_and_capacity_errors_launch_nothing(qsa):
    lib = ctypes.CDLL(qsa.LIB_PATH)
    lib.qsa_compress_keys.restype = ctypes.c_int
    cfg = qsa.Config().c()
    # NULL idx_k -> INVALID_ARG before any CUDA call.
    st = lib.qsa_compress_keys(ctypes.byref(cfg), 1, None, ctypes.c_int64(64), None, ctypes.c_int64(0),
                               ctypes.c_int64(1), ctypes.c_void_p(256), None)
    assert st == 1
    # Block range past the capacity -> CAPACITY (fake, aligned, never dereferenced pointers).
    st = lib.qsa_compress_keys(ctypes.byref(cfg), 1, ctypes.c_void_p(4096), ctypes.c_int64(64), None,
                               ctypes.c_int64(0), ctypes.c_int64(17), ctypes.c_void_p(8192), None)
    assert st == 4
    lib.qsa_last_error.restype = ctypes.c_char_p
    assert b"cap" in lib.qsa_last_error()


def test_fault_injection_arguments_are_validated(qsa):
    """Host-side checks of the failure-path switch (no device work)."""
    for mode, wait, ok in [(5, 0.1, False), (-1, 0.1, False), (1, 0.0, False), (1, 11.0, False),
                           (1, float("nan"), False), (2, 0.0, False), (3, 0.0, False), (4, 0.0, False),
                           (4, 10.5, False), (1, 0.5, True), (2, 0.5, True), (3, 0.5, True), (4, 0.5, True),
                           (0, 0.0, True)]:
        if ok:
            qsa.qsa_set_fault_injection(mode, wait)
        else:
            with pytest.raises(qsa.QSAError) as e:
                qsa.qsa_set_fault_injection(mode, wait)
            assert e.value.status == 1, (mode, wait)
    qsa.qsa_set_fault_injection(0)


def test_quantize_rows_validation_launches_nothing(qsa):
    lib = ctypes.CDLL(qsa.LIB_PATH)
    lib.qsa_quantize_rows.restype = ctypes.c_int
    lib.qsa_quantize_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]
    p = ctypes.c_void_p(4096)  # aligned, never dereferenced
    assert lib.qsa_quantize_rows(p, 10, 96, p, p, None) == 2  # dim not 64/128/256: unsupported
    assert lib.qsa_quantize_rows(None, 10, 128, p, p, None) == 1
    assert lib.qsa_quantize_rows(p, 10, 128, p, ctypes.c_void_p(4098), None) == 1  # scales misaligned
    assert lib.qsa_quantize_rows(p, 0, 128, p, p, None) == 0  # nothing to do


def test_binding_argument_counts_match_the_header(qsa):
    """Every ctypes signature of the binding has as many arguments as the
    declaration in include/qsa.h."""
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    decls = {m.group(1): m.group(2) for m in re.finditer(r"\b(qsa_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", src)}
    for name, args in qsa._SIGS.items():
        assert name in decls, name
        params = [p for p in decls[name].split(",") if p.strip() and p.strip() != "void"]
        assert len(args) == len(params), (name, len(args), len(params))


def test_training_entry_points_validate_before_launching(qsa):
    """The backward, distillation-target and KL calls reject bad arguments with
    a status and launch nothing (fake, aligned, never dereferenced pointers)."""
    lib = ctypes.CDLL(qsa.LIB_PATH)
    for name in ("qsa_sparse_attention_backward", "qsa_distill_target", "qsa_distill_kl"):
        getattr(lib, name).restype = ctypes.c_int
        getattr(lib, name).argtypes = qsa._SIGS[name]
    cfg = ctypes.byref(qsa.Config().c())
    p = ctypes.c_void_p(4096)
    bwd = lib.qsa_sparse_attention_backward
    assert bwd(cfg, 1, p, 0, 16, p, p, 64, p, p, p, None, p, p, p, p, None) == 1  # lse is required
    assert bwd(cfg, 1, p, 60, 16, p, p, 64, p, p, p, p, p, p, p, p, None) == 4  # queries past cap
    assert bwd(cfg, 1, p, 0, 16, p, p, 64, p, p, p, p, p, None, p, p, None) == 1  # dq NULL
    assert bwd(cfg, 1, p, 0, 0, p, p, 64, p, p, p, p, p, p, p, p, None) == 0  # nothing to do
    tgt = lib.qsa_distill_target
    big = 1 << 20
    assert tgt(cfg, 1, p, 0, 64, p, 64, p, 8, p, big, None) == 1  # ld < floor(63 / 4)
    assert tgt(cfg, 1, p, 0, 64, p, 32, p, 16, p, big, None) == 4  # queries past cap
    assert tgt(ctypes.byref(qsa.Config(r=3).c()), 1, p, 0, 8, p, 64, p, 16, p, big, None) == 2  # r not in {1..16}
    assert tgt(ctypes.byref(qsa.Config(q_heads=64, kv_heads=4).c()), 1, p, 0, 8, p, 64, p, 16, p, big, None) == 2
    assert tgt(cfg, 1, p, 0, 64, p, 64, p, 16, p, 256, None) == 3  # workspace without the lse rows
    assert tgt(cfg, 4096, p, 0, 64, p, 1 << 20, p, 16, p, big, None) == 2  # batch x cap past 32-bit rows
    assert tgt(cfg, 1, p, 0, 0, p, 64, p, 0, None, 0, None) == 0
    assert qsa.qsa_workspace_size(qsa.Config(), qsa.OP_DISTILL_TARGET, 2, 64, 10) == 256 + 2 * 10 * 32 * 4
    kl = lib.qsa_distill_kl
    assert kl(cfg, 1, 0, 64, p, p, 8, p, None, None) == 1  # ld too small
    assert kl(cfg, 1, 0, 64, p, p, 16, ctypes.c_void_p(4098), None, None) == 1  # kl misaligned
    assert kl(cfg, 1, 0, 0, p, p, 0, p, None, None) == 0


def test_offload_decode_validates_before_launching(qsa):
    """qsa_decode_step_offload rejects a bad hot-cache size and host caches that
    are not pinned, mapped host memory (fake, aligned, never dereferenced
    pointers), with a status and no launch."""
    lib = ctypes.CDLL(qsa.LIB_PATH)
    f = lib.qsa_decode_step_offload
    f.restype = ctypes.c_int
    f.argtypes = qsa._SIGS["qsa_decode_step_offload"]
    cfg = ctypes.byref(qsa.Config().c())
    p = ctypes.c_void_p(4096)
    lib.qsa_last_error.restype = ctypes.c_char_p
    lib.qsa_launch_count.restype = ctypes.c_uint64
    n0 = lib.qsa_launch_count()

    def call(hot_blocks):
        # cfg, batch, pos, q, k, v, idx_q, idx_k, host_k, host_v, hot_k, hot_v, hot_tags, hot_blocks,
        # idx_k_cache, pooled, cap, rms_w, out, sel, nsel, ws, ws_bytes, stream
        return f(cfg, 1, p, p, p, p, p, p, p, p, p, p, p, hot_blocks, p, p, 4096, None, p, None, None, p,
                 1 << 20, None)

    assert call(0) == 1 and call(2 ** 31 - 1) == 1  # hot_blocks outside [1, INT32_MAX)
    assert call(64) == 1                            # the host caches are not mapped host memory
    assert b"host" in lib.qsa_last_error()
    assert lib.qsa_launch_count() == n0


def test_attention_kernel_switch_is_validated(qsa):
    """Host-side check of the sparse-attention kernel switch (no device work)."""
    for k in (0, 1):
        qsa.qsa_set_attention_kernel(k)
    for k in (-1, 2):
        with pytest.raises(qsa.QSAError) as e:
            qsa.qsa_set_attention_kernel(k)
        assert e.value.status == 1
    qsa.qsa_set_attention_kernel(0)


def test_decode_kernel_switch_is_validated(qsa):
    """Host-side check of the decode-step kernel switch (no device work)."""
    for k in (qsa.DECODE_THREE_KERNELS, qsa.DECODE_STEP_KERNEL):
        qsa.qsa_set_decode_kernel(k)
    for k in (-1, 2):
        with pytest.raises(qsa.QSAError) as e:
            qsa.qsa_set_decode_kernel(k)
        assert e.value.status == 1
    qsa.qsa_set_decode_kernel(1)
