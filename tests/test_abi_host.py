"""Host-side checks of the C ABI (no GPU needed, no compute calls).

libwq.so must load, export every function include/wq.h declares, and its
host-only entry points (status strings, sizes, tuning-file parsing) must
behave as documented.
"""
import ctypes
import os
import subprocess
import sys

import pytest

import weight_only_quantized_02_b200 as wq


def test_library_exports_every_header_symbol():
    names = wq.header_functions()
    assert "wq_linear" in names and "wq_pack_int4" in names and "wq_pack_int8" in names
    missing = [n for n in names if not hasattr(wq.lib, n)]
    assert not missing, missing


def test_binding_covers_every_header_symbol():
    missing = [n for n in wq.header_functions() if not callable(getattr(wq, n, None))]
    assert not missing, missing


def test_exports_with_nm():
    out = subprocess.run(["nm", "-D", "--defined-only", wq.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for n in wq.header_functions():
        assert n in exported, n


def test_strerror_is_defined_for_every_status():
    for code in list(wq.STATUS) + [-99, 7]:
        s = wq.strerror(code)
        assert isinstance(s, str) and s
    assert wq.strerror(0) == "ok"


def test_packed_bytes():
    wb, sb, zb = wq.wq_packed_bytes(8, 5120, 17408, 0)
    assert wb == 5120 * 17408 + 64 and sb == 17408 * 2 and zb == 0
    wb, sb, zb = wq.wq_packed_bytes(4, 5120, 25600, 128)
    assert wb == 5120 * 25600 // 2 + 64
    assert sb == 25600 * 40 * 2 and zb == 25600 * 40 // 2
    # ragged: N not a multiple of the 128-row panel, K not a multiple of the 128-k block
    wb, sb, zb = wq.wq_packed_bytes(8, 1120, 400, 0)
    assert wb == 512 * 1152 + 64 and sb == 512 * 2
    # INT4 groups of 32 and 64 k: one scale and zero point per group; per-channel
    # (group = K) is stored as group 128 with the row's pair repeated
    for g in (32, 64):
        wb, sb, zb = wq.wq_packed_bytes(4, 5120, 25600, g)
        assert wb == 5120 * 25600 // 2 + 64 and sb == 25600 * (5120 // g) * 2 and zb == 25600 * (5120 // g) // 2
    assert wq.wq_packed_bytes(4, 5120, 25600, 5120) == wq.wq_packed_bytes(4, 5120, 25600, 128)


@pytest.mark.parametrize("bits,K,N,group,status", [
    (8, 1024, 1024, 128, -4),   # INT8 takes no group
    (4, 1024, 1024, 48, -4),    # groups: 32, 64, 128 or K
    (4, 1024, 1024, 256, -4),   # neither a listed group nor K
    (4, 1000, 1024, 128, -2),   # K not a multiple of the group
    (8, 1000, 1024, 0, -2),     # K not a multiple of 32
    (8, 1040, 1024, 0, -2),     # INT8: K % 32 (a multiple of 16 is not enough: 32-k integer MMA steps)
    (8, 1024, 1000, 0, -2),     # N not a multiple of 16 (a multiple of 8 is not enough: 16-row blocks)
    (8, 32, (1 << 20) + 16, 0, -2),  # N beyond the workspace's fixed counter region (2^20 channels)
    (8, 0, 1024, 0, -2),
    (3, 1024, 1024, 0, -4),
])
def test_packed_bytes_rejects(bits, K, N, group, status):
    a = ctypes.c_size_t()
    assert wq.lib.wq_packed_bytes(bits, K, N, group, ctypes.byref(a), None, None) == status


def test_workspace_bytes():
    # counters: a region of one size for every shape -- 8 tickets per
    # 128-row panel of the largest N (2^20: 8192 panels) + 2 grid counters +
    # 64 two-word residual sums of the integer path's exactness guard, padded
    # to 256 bytes (65666 words -> 262912 bytes); then the largest of the
    # split-K GEMM's fp32 partials [S][M][N], the stream-K kernels' per-CTA
    # panel partials [512 CTAs][2][128 rows][token tile] and the integer
    # path's digits + int32 partials (smaller than the stream-K GEMM's here)
    C = 262912
    assert wq.wq_workspace_bytes(128, 5120, 5120, 32) == C + 32 * 128 * 5120 * 4
    assert wq.wq_workspace_bytes(64, 5120, 5120, 1) == C + 512 * 2 * 128 * 64 * 4
    # M = 16: the integer tensor-core GEMM's digit blocks (40 k-blocks x 48 digit rows x 128) and int32
    # partials [2 CTAs per SM x 160][2][48][128]
    assert wq.wq_workspace_bytes(16, 5120, 5120, 1) == C + 40 * 48 * 128 + 320 * 2 * 48 * 128 * 4
    # M = 8: the integer GEMV's per-warp partials 448 CTAs x 8 warps x 2 x 16 rows x 24 x 4 bytes
    assert wq.wq_workspace_bytes(8, 5120, 5120, 1) == C + 448 * 8 * 2 * 16 * 24 * 4
    assert wq.wq_workspace_bytes(1, 5120, 17408, 1) == C + 512 * 2 * 128 * 16 * 4
    # integer path, M = 1 (16 digit rows): int32 partials 160 CTAs x 2 x 16 x 128
    assert 160 * 2 * 16 * 128 * 4 < 512 * 2 * 128 * 16 * 4
    assert wq.wq_workspace_bytes(0, 5120, 5120, 4) == 0
    assert wq.wq_workspace_bytes(1, 0, 5120, 4) == 0


def test_topk_workspace_bytes():
    # the bf16 logits M x N (padded to 256 bytes), then P candidates of k
    # 64-bit (key, index) words per token; P slices of 4096 logits, or of
    # 8192 when the 4096-logit grid (P x M CTAs) would not fit the GPU at
    # once (4 CTAs x 148 SMs = 592)
    def expect(M, N, k, S):
        P = -(-N // S)
        return -(-(M * N * 2) // 256) * 256 + M * P * k * 8
    V = 152064  # the vocabulary head: 38 slices of 4096, or 19 of 8192
    assert wq.wq_topk_workspace_bytes(1, V, 64) == expect(1, V, 64, 4096) == 304128 + 38 * 64 * 8
    assert wq.wq_topk_workspace_bytes(4, V, 64) == expect(4, V, 64, 4096)
    assert wq.wq_topk_workspace_bytes(15, V, 64) == expect(15, V, 64, 4096)  # 570 CTAs: one wave
    assert wq.wq_topk_workspace_bytes(16, V, 64) == expect(16, V, 64, 8192)  # 608 CTAs: wider slices
    assert wq.wq_topk_workspace_bytes(128, V, 1) == expect(128, V, 1, 8192)
    assert wq.wq_topk_workspace_bytes(1, 1, 1) == 256 + 8
    assert wq.wq_topk_workspace_bytes(2, 4097, 3) == 256 * 65 + 2 * 2 * 3 * 8  # a ragged last slice
    # outside the limits: no scratch
    assert wq.wq_topk_workspace_bytes(0, V, 64) == 0
    assert wq.wq_topk_workspace_bytes(1, V, 65) == 0  # k > 64
    assert wq.wq_topk_workspace_bytes(1, 8, 9) == 0   # k > N
    assert wq.wq_topk_workspace_bytes(1, V, 0) == 0
    # the merge keeps P k candidates (two 32-bit words each) in shared memory, at most 200 KB
    assert wq.wq_topk_workspace_bytes(1, 367 * 4096, 64) == expect(1, 367 * 4096, 64, 4096)
    assert wq.wq_topk_workspace_bytes(1, 368 * 4096, 64) == 0


def test_null_pointer_checks_need_no_device():
    assert wq.lib.wq_linear(None, 1, 1024, None, None, None, 0, 1024, None, None) == -1
    assert wq.lib.wq_pack_int8(None, None, 1024, 1024, None, None, None) == -1
    assert wq.lib.wq_quantize_int4(None, 1024, 16, 128, None, None, None, None) == -1


def test_topk_argument_checks_need_no_device():
    # every check of wq_linear_topk runs before its first CUDA call; the
    # pointers here are never dereferenced
    f = wq.lib.wq_linear_topk
    P = ctypes.c_void_p
    x, w, s, z, v, i = (P(0x10000 * n) for n in range(1, 7))
    ws = P(0x100000)
    V = 152064
    need = wq.wq_topk_workspace_bytes(4, V, 64)

    def call(M=4, N=V, k=64, vals=v, idx=i, scratch=ws, nbytes=need):
        return f(x, M, 5120, w, s, z, 0, N, k, vals, idx, scratch, nbytes, None)
    for kw in (dict(M=0), dict(M=129), dict(k=0), dict(k=65), dict(N=32, k=33), dict(M=1, N=368 * 4096)):
        assert call(**kw) == -2, kw  # WQ_ERR_SHAPE
    assert call(vals=None) == -1 and call(idx=None) == -1 and call(scratch=None) == -1  # WQ_ERR_NULL
    assert call(scratch=P(0x100008)) == -3  # WQ_ERR_ALIGN: the scratch must be 16-byte aligned
    assert call(nbytes=need - 1) == -6  # WQ_ERR_WORKSPACE


def test_tuning_file_parse_errors(tmp_path):
    good = tmp_path / "good.txt"
    good.write_text("# comment\nNVIDIA B200|148 1 5120 17408 8 0 0 4 12.500\n"
                    "NVIDIA B200|148 4 5120 17408 8 0 4 1 9.000\n"
                    "NVIDIA B200|148 2 5120 25600 4 128 5 2 20.000\n")
    assert wq.wq_load_tuning(str(good)) == 0
    for bad_line in [
        "NVIDIA B200|148 1 5120 17408 8 0 2 3 12.5\n",      # row-block GEMV split must be 1/2/4/8
        "NVIDIA B200|148 1 5120 17408 8 0 0 5 12.5\n",      # stream-K GEMV: 1..4 CTAs per SM
        "NVIDIA B200|148 200 5120 17408 8 0 1 4 12.5\n",    # M > 128
        "NVIDIA B200|148 1 5120 17408 8 64 0 4 12.5\n",     # bad group
        "NVIDIA B200 1 5120 17408 8 0 0 4 12.5\n",          # no device key separator
        "NVIDIA B200|148 1 5120 17408 8 0 0\n",             # truncated
        "NVIDIA B200|148 1 5120 17408 8 0 0 4 12.5 extra\n",
        "NVIDIA B200|148 64 17408 5120 4 128 1 64 1.0\n",   # split above 32
        "NVIDIA B200|148 65 5120 17408 8 0 4 1 9.0\n",      # integer path: M <= 64
        "NVIDIA B200|148 33 5120 17408 4 128 4 1 9.0\n",    # integer path, W4A16: M <= 32
        "NVIDIA B200|148 4 5120 17408 8 0 4 2 9.0\n",       # integer path: split 1 only
        "NVIDIA B200|148 9 5120 17408 8 0 5 1 9.0\n",       # integer GEMV: M <= 8
        "NVIDIA B200|148 8 65536 17408 8 0 5 1 9.0\n",      # integer GEMV: digit rows over 200 KB
        "NVIDIA B200|148 4 5120 17408 4 128 5 3 9.0\n",     # integer GEMV: split 1 or 2
        "NVIDIA B200|148 16 17408 5120 8 0 6 1 9.0\n",      # role-split GEMM: W4A16 only
        "NVIDIA B200|148 16 17408 5120 4 128 6 2 9.0\n",    # role-split GEMM: split 1 only
    ]:
        p = tmp_path / "bad.txt"
        p.write_text(bad_line)
        assert wq.wq_load_tuning(str(p)) == -8, bad_line
    assert wq.wq_load_tuning(str(tmp_path / "missing.txt")) == -8
    assert wq.lib.wq_load_tuning(None) == -1


def test_shipped_tuning_table_loads():
    """The measured B200 table that ships with the package parses and holds
    only valid (variant, split) choices."""
    path = os.path.join(os.path.dirname(wq.__file__), "tuning_b200.txt")
    assert wq.wq_load_tuning(path) == 0
    entries = [l for l in open(path) if "|" in l and not l.startswith("#")]
    assert len(entries) >= 14
    wq.wq_clear_tuning()


def test_no_oracle_in_product():
    """The product package never imports or links the oracle."""
    here = os.path.dirname(wq.__file__)
    for root, _, files in os.walk(here):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(root, f)).read()
                assert "import oracle" not in text and "from oracle" not in text and "liboracle" not in text, f


def _run_with_env(code, env_extra):
    env = dict(os.environ)
    env.update(env_extra)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=root, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    return out.stdout


def test_tuning_file_from_environment_is_loaded(tmp_path):
    shipped = os.path.join(os.path.dirname(wq.__file__), "tuning_b200.txt")
    saved = tmp_path / "saved.txt"
    _run_with_env(f"import weight_only_quantized_02_b200 as wq; assert wq.lib.wq_save_tuning({str(saved)!r}.encode()) == 0",
                  {"WQ_TUNING_FILE": shipped})

    def entries(path):
        return sorted(" ".join(l.split()[:9]) for l in open(path) if l.strip() and not l.startswith("#"))

    assert entries(saved) == entries(shipped)


def test_unreadable_tuning_file_from_environment_fails_automatic_choices(tmp_path):
    code = ("import ctypes, weight_only_quantized_02_b200 as wq\n"
            "v, s = ctypes.c_int(0), ctypes.c_int(0)\n"
            "print(wq.lib.wq_get_choice(1, 5120, 17408, 8, 0, ctypes.byref(v), ctypes.byref(s)))\n")
    out = _run_with_env(code, {"WQ_TUNING_FILE": str(tmp_path / "missing.txt")})
    assert int(out.strip().splitlines()[-1]) == -8  # WQ_ERR_TUNING
    bad = tmp_path / "bad.txt"
    bad.write_text("this is not a table\n")
    out = _run_with_env(code, {"WQ_TUNING_FILE": str(bad)})
    assert int(out.strip().splitlines()[-1]) == -8
