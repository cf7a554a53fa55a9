"""The C ABI from plain C: include/tp_block.h compiles as C99 and a C program links
against libtp_block.so and calls the host-only entry points (CPU only)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_header_and_library_from_c(tmp_path):
    import tensor_llama_transformer_b200 as tpb

    libdir = os.path.dirname(tpb.LIB_PATH)
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), "-L", libdir, "-ltp_block",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    assert "sm_100a" in got["version"] and got["status_ok"] == "ok"
    assert got["block_ws_rc"] == str(tpb.TP_OK)
    assert int(got["block_ws"]) == tpb.tp_block_workspace_bytes(
        tpb.make_dims(4096, 32, 32, 128, 11008, 32000, 1, 1024), 4, tpb.TP_PART_1D, 1)
    assert got["rank_ws_rc"] == str(tpb.TP_OK) and 0 < int(got["rank_ws"]) < int(got["block_ws"])
    assert got["bad_slices_rc"] == str(tpb.TP_EINVAL)
    assert got["create_no_ws_rc"] == str(tpb.TP_EINVAL)  # NULL weights
    assert got["quantize_bad_n_rc"] == str(tpb.TP_EINVAL)
