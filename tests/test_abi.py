"""C-ABI checks that need no GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching any
device.  All pointers passed here are rejected by host-side validation, so
nothing is ever launched."""
import ctypes

import pytest
import torch

from tensor_core_gemm_fp16_b200 import binding

NONE, BIAS, GELU = 0, 1, 2


# Tests marked no_device_only pass made-up device addresses that host validation must reject
# before any device call.  They run only where no CUDA device exists, so a
# regression in the validation can never reach a GPU with those addresses.
no_device_only = pytest.mark.skipif(torch.cuda.is_available(),
                                    reason="made-up addresses: host-only check")


def test_library_exports_every_header_symbol():
    lib = binding.load()
    names = binding.header_symbols()
    assert "tg_gemm" in names and "tg_gemm_check_error" in names
    assert "tg_attention_fwd" in names and "tg_attention_fwd_ex" in names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/*.h but not exported"


@no_device_only
def test_attention_host_validation_without_a_device():
    """Every call here is rejected on the host before any device query."""
    f = binding.tg_attention_fwd
    q, k, v, o = 0x100000, 0x200000, 0x300000, 0x400000
    bad = binding.TG_ERR_INVALID_ARG
    assert f(q, k, v, o, 1, 1, 128, 128, 96, 0, 0.0) == bad            # head_dim
    assert f(q, k, v, o, 1, 1, 128, 128, 64, 2, 0.0) == bad            # causal flag
    assert f(q, k, v, o, -1, 1, 128, 128, 64, 0, 0.0) == bad           # negative size
    assert f(q, k, v, o, 1, 1, 128, 128, 64, 0, float("nan")) == bad   # scale
    assert f(None, k, v, o, 1, 1, 128, 128, 64, 0, 0.0) == bad         # null pointer
    assert f(q, k, v, q + 64, 1, 1, 128, 128, 64, 0, 0.0) == bad       # O overlaps Q
    assert f(q + 8, k, v, o, 1, 1, 128, 128, 64, 0, 0.0) == binding.TG_ERR_MISALIGNED
    assert f(q, k, v, o, 0, 4, 128, 128, 64, 0, 0.0) == binding.TG_OK   # empty: no-op
    assert binding.tg_attention_fwd_ex(q, k, v, o, 1, 1, 8, 8, 64, 0, 0.0, inject=9) == bad
    assert binding.tg_attention_fwd_ex(q, k, v, o, 1, 1, 8, 8, 64, 0, 0.0, kv_split=3) == bad
    assert binding.tg_attention_fwd_ex(q, k, v, o, 1, 1, 8, 8, 64, 0, 0.0, kv_split=-1) == bad


def test_status_strings():
    for st in range(8):
        s = binding.tg_status_string(st)
        assert s.startswith("TG_")
    assert "unknown" in binding.tg_status_string(99)


def test_config_table_is_consistent():
    n = binding.tg_num_configs()
    assert n >= 3
    ids = set()
    for i in range(n):
        c = binding.tg_config_info(i)
        assert c["id"] == i
        ids.add(i)
        assert c["block_m"] == 128 * (2 if c["cta_pair"] else 1)
        assert c["block_n"] in (64, 128, 256)
        assert c["block_k"] in (64, 128)
        assert 2 <= c["stages"] <= 12
        assert c["group_m"] >= 1
    with pytest.raises(binding.TgError):
        binding.tg_config_info(n)
    with pytest.raises(binding.TgError):
        binding.tg_config_info(-1)


@pytest.mark.parametrize("M,N,K", [(256, 256, 256), (2048, 2048, 2048), (3000, 1537, 2050),
                                   (8192, 8192, 8192), (1, 1, 1), (100000, 64, 64)])
def test_select_config_is_host_only_and_valid(M, N, K):
    c = binding.tg_gemm_select_config(M, N, K, GELU, 148)
    assert 0 <= c["id"] < binding.tg_num_configs()


def test_select_config_prefers_more_tiles_for_small_problems():
    small = binding.tg_gemm_select_config(256, 256, 256, NONE, 148)
    big = binding.tg_gemm_select_config(8192, 8192, 8192, GELU, 148)
    assert small["block_n"] <= big["block_n"]


def test_select_config_reports_the_split():
    """Whole tiles when there are enough of them; stream-K for a deep
    contraction with fewer tiles than SMs; never stream-K for the softmax."""
    assert binding.tg_gemm_select_config(8192, 8192, 8192, GELU, 148)["split"] == \
        binding.TG_SPLIT_TILES
    assert binding.tg_gemm_select_config(512, 512, 16384, NONE, 148)["split"] == \
        binding.TG_SPLIT_STREAM_K
    assert binding.tg_gemm_select_config(1024, 1024, 8192, GELU, 148)["split"] == \
        binding.TG_SPLIT_STREAM_K
    assert binding.tg_gemm_select_config(256, 256, 256, NONE, 148)["split"] == \
        binding.TG_SPLIT_TILES
    assert binding.tg_gemm_select_config(8192, 256, 65536, 4, 148)["split"] == \
        binding.TG_SPLIT_TILES
    assert binding.tg_config_info(0)["split"] == 0


def test_select_config_rejects_bad_args():
    with pytest.raises(binding.TgError):
        binding.tg_gemm_select_config(-1, 4, 4, NONE, 148)
    with pytest.raises(binding.TgError):
        binding.tg_gemm_select_config(4, 4, 4, 5, 148)
    with pytest.raises(binding.TgError):
        binding.tg_gemm_select_config(4, 4, 4, 0, 0)


@no_device_only
def test_host_validation_rejects_bad_calls_without_a_device():
    g = binding.tg_gemm
    # bad epilogue
    assert g(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 7, None) == binding.TG_ERR_INVALID_ARG
    # negative and oversized dimensions
    assert g(0x1000, 0x2000, None, 0x30000, -1, 4, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    assert g(0x1000, 0x2000, None, 0x30000, 4, 1 << 31, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    # null C / null A with K > 0
    assert g(0x1000, 0x2000, None, None, 4, 4, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    assert g(None, 0x2000, None, 0x30000, 4, 4, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    # odd addresses
    assert g(0x1001, 0x2000, None, 0x30000, 4, 4, 4, 0, None) == binding.TG_ERR_MISALIGNED
    assert g(0x1000, 0x2000, 0x5001, 0x30000, 4, 4, 4, 1, None) == binding.TG_ERR_MISALIGNED
    # C overlapping A, B or bias
    assert g(0x10000, 0x20000, None, 0x10010, 4, 4, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    assert g(0x10000, 0x20000, None, 0x1FFF8, 4, 4, 4, 0, None) == binding.TG_ERR_INVALID_ARG
    assert g(0x10000, 0x20000, 0x40004, 0x40000, 4, 4, 4, 1, None) == binding.TG_ERR_INVALID_ARG
    # bad options
    assert binding.tg_gemm_ex(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 9) == binding.TG_ERR_INVALID_ARG
    assert binding.tg_gemm_ex(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 0, config_id=99) == \
        binding.TG_ERR_INVALID_ARG
    assert binding.tg_gemm_ex(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 0, group_m=65) == \
        binding.TG_ERR_INVALID_ARG
    assert binding.tg_gemm_ex(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 0, inject=7) == \
        binding.TG_ERR_INVALID_ARG
    assert binding.tg_gemm_ex(0x1000, 0x2000, None, 0x30000, 4, 4, 4, 0, split=3) == \
        binding.TG_ERR_INVALID_ARG


def test_empty_problems_are_ok_without_a_device():
    assert binding.tg_gemm(None, None, None, None, 0, 4, 4, 0, None) == binding.TG_OK
    assert binding.tg_gemm(None, None, None, None, 4, 0, 4, 2, None) == binding.TG_OK


@no_device_only
def test_host_entry_validation():
    lib = binding
    need = lib.tg_gemm_host_workspace_size(10, 20, 30, True)
    assert need == 768 + 1280 + 256 + 512   # 600, 1200, 40, 400 bytes, each rounded to 256
    assert lib.tg_gemm_host_workspace_size(-1, 2, 3, False) == 0
    # workspace too small / misaligned
    assert lib.tg_gemm_host(0x1000, 0x20000, None, 0x40000, 10, 20, 30, 0, 0x100000, 10) == \
        binding.TG_ERR_INVALID_ARG
    assert lib.tg_gemm_host(0x1000, 0x20000, None, 0x40000, 10, 20, 30, 0, 0x100010, need) == \
        binding.TG_ERR_INVALID_ARG


@no_device_only
def test_noalloc_scratch_limit_is_checked_on_the_host():
    # K = 127 repacks A into 128-element rows (256 bytes each): 131072 rows
    # need exactly TG_NOALLOC_SCRATCH_BYTES and pass the size check (then
    # find no device); one row more needs 256 bytes more and is rejected.
    limit = binding.noalloc_scratch_bytes()
    M = limit // 256
    f = binding.tg_gemm_noalloc
    assert f(0x1000000, 0x100000000, None, 0x200000000, M, 8, 127, 0, None) == \
        binding.TG_ERR_UNSUPPORTED_DEVICE
    st = f(0x1000000, 0x100000000, None, 0x200000000, M + 1, 8, 127, 0, None)
    assert st == binding.TG_ERR_SCRATCH_LIMIT
    # B repacked alone: K * N8 * 2 bytes (N = 1023 -> 1024-element rows)
    assert f(0x1000000, 0x100000000, None, 0x200000000, 8, 1023, limit // 2048, 0, None) == \
        binding.TG_ERR_UNSUPPORTED_DEVICE
    assert f(0x1000000, 0x100000000, None, 0x200000000, 8, 1023, limit // 2048 + 1, 0, None) == \
        binding.TG_ERR_SCRATCH_LIMIT


@no_device_only
def test_valid_call_without_a_device_reports_unsupported_device():
    # Passes host validation, then finds no sm_100 device: nothing runs.
    st = binding.tg_gemm(0x100000, 0x200000, None, 0x300000, 4, 4, 4, 0, None)
    assert st == binding.TG_ERR_UNSUPPORTED_DEVICE
    assert binding.tg_gemm_check_error(None) == binding.TG_ERR_UNSUPPORTED_DEVICE


def test_launch_count_is_host_only():
    """One GEMM kernel, plus one repacking kernel for both operands when
    either row pitch or base is not a multiple of 16 bytes (it also gathers the
    thin remainder's columns of B), plus the thin N-remainder kernel when it
    saves the GEMM a wave."""
    f = binding.tg_gemm_launch_count
    assert f(0x1000, 0x100000, None, 0x1000000, 256, 256, 256, NONE) == 1
    assert f(0x1000, 0x100000, None, 0x1000000, 256, 256, 250, NONE) == 2   # K % 8
    assert f(0x1000, 0x100000, None, 0x1000000, 256, 250, 256, NONE) == 2   # N % 8
    assert f(0x1000, 0x100000, None, 0x1000000, 300, 1537, 2050, GELU) == 2  # both
    # 3000 x 1537: the last column of 256-wide tiles (one valid column) would
    # add a second wave; the tail kernel computes that column instead
    assert f(0x1000, 0x100000, None, 0x1000000, 3000, 1537, 2050, GELU) == 3
    assert f(0x1002, 0x100000, None, 0x1000000, 256, 256, 256, NONE) == 2   # A's base
    assert f(0x1000, 0x100000, None, 0x1000000, 256, 256, 0, GELU) == 1     # K == 0
    assert f(0x1000, 0x100000, None, 0x1000000, 0, 256, 256, NONE) == 0
    assert f(0x1001, 0x100000, None, 0x1000000, 256, 256, 256, NONE) == -1  # misaligned


def test_binding_checks_tensor_arguments():
    a = torch.zeros(4, 4, dtype=torch.float32)
    with pytest.raises(TypeError):
        binding.gemm(a, a)
    h = torch.zeros(4, 4, dtype=torch.float16)
    with pytest.raises(ValueError):
        binding.gemm(h, h)          # not CUDA tensors


@no_device_only
def test_softmax_limits_are_checked_on_the_host():
    assert binding.tg_gemm(0x1000, 0x200000, None, 0x400000, 4, 257, 4, 4, None) == \
        binding.TG_ERR_INVALID_ARG
    with pytest.raises(binding.TgError):
        binding.tg_gemm_select_config(100, 300, 64, 4, 148)
    c = binding.tg_gemm_select_config(100, 200, 64, 4, 148)
    assert c["epi_warps"] == 4 and c["block_n"] >= 200
    assert binding.tg_gemm(0x1000, 0x200000, None, 0x400000, 4, 4, 4, 5, None) == \
        binding.TG_ERR_INVALID_ARG


def test_attention_plan_without_a_device():
    """The work division of the attention launch, as a host-only query: one
    unit per (batch x head, 256 queries); a non-causal last wave that fills at
    most half of the SMs is split into key halves; never for causal calls or a
    single key tile; forced or disabled by kv_split."""
    plan = binding.tg_attention_plan
    assert plan(4, 16, 2048, 2048, 128, False) == {"units": 512, "split": 68, "grid": 580}
    assert plan(4, 16, 2048, 2048, 64, True) == {"units": 512, "split": 0, "grid": 512}
    assert plan(4, 16, 2048, 2048, 128, False, kv_split=binding.TG_ATTN_SPLIT_NEVER)["split"] == 0
    assert plan(1, 2, 256, 256, 64, False) == {"units": 2, "split": 2, "grid": 4}
    assert plan(1, 2, 256, 128, 64, False)["split"] == 0                  # one key tile
    assert plan(1, 2, 256, 128, 64, False, kv_split=binding.TG_ATTN_SPLIT_ALL)["split"] == 0
    assert plan(2, 3, 200, 333, 64, False, kv_split=binding.TG_ATTN_SPLIT_ALL) == \
        {"units": 6, "split": 6, "grid": 12}
    assert plan(1, 296, 256, 512, 64, False)["split"] == 0                # two full waves
    assert plan(1, 248, 256, 512, 64, False)["split"] == 0                # last wave 100 > 74
    assert plan(1, 222, 256, 512, 64, False)["split"] == 74               # last wave 74
    assert plan(1, 8, 1000, 512, 64, False, num_sms=16) == {"units": 32, "split": 0, "grid": 32}
    assert plan(1, 9, 1000, 512, 64, False, num_sms=16) == {"units": 36, "split": 4, "grid": 40}
    assert plan(0, 4, 128, 128, 64, False) == {"units": 0, "split": 0, "grid": 0}
    assert plan(1, 1, 128, 0, 64, False) == {"units": 0, "split": 0, "grid": 0}
    for bad in ({"head_dim": 96}, {"kv_split": 3}, {"num_sms": 0}, {"causal": 2}):
        args = {"batch": 1, "heads": 1, "seq_q": 128, "seq_k": 128, "head_dim": 64,
                "causal": 0, "kv_split": 0, "num_sms": 148}
        args.update(bad)
        with pytest.raises(binding.TgError):
            plan(**args)


def test_plain_c_client_compiles_links_and_runs(tmp_path):
    """Both public headers compile as strict C99, and a C program linked
    against the library runs its host-only entry points (no GPU needed)."""
    import os
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(binding.LIB_PATH)
    exe = tmp_path / "abi_client"
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(root, "include"),
                    os.path.join(root, "tests", "c_client", "abi_client.c"),
                    "-L", libdir, "-ltg_gemm", f"-Wl,-rpath,{libdir}", "-o", str(exe)],
                   check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "attention plan: units 512 split 68 grid 580" in out.stdout
    assert out.stdout.strip().endswith("OK")
