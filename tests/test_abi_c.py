"""The C ABI from C (CPU only): a plain C client (tests/c_abi_client.c) is compiled
against include/*.h, linked to libpagedattn.so and run; its view of the host-side
entry points must agree with the Python binding, the xxhash package and the
block-manager oracle.  The same client also compiles as C++."""
import subprocess
from pathlib import Path

import pytest
import xxhash

from oracle.block_manager import OracleBlockManager

ROOT = Path(__file__).resolve().parent.parent
PKG = ROOT / "paged_kv_cache_331_b200"


@pytest.fixture(scope="module")
def client_output(tmp_path_factory):
    from paged_kv_cache_331_b200 import build as B
    B.build()
    exe = tmp_path_factory.mktemp("c_abi") / "client"
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", f"-I{ROOT / 'include'}",
                    str(ROOT / "tests" / "c_abi_client.c"), f"-L{PKG}", "-lpagedattn", f"-Wl,-rpath,{PKG}",
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, check=True)
    return {line.split()[0]: line.split()[1:] for line in r.stdout.splitlines() if line.strip()
            if not line.startswith("status ")} | \
        {"status": [line.split()[1:] for line in r.stdout.splitlines() if line.startswith("status ")]}


def test_headers_compile_as_cxx(tmp_path):
    """The same client compiled as C++ (the headers' extern "C" guards) links and prints the same lines."""
    from paged_kv_cache_331_b200 import build as B
    B.build()
    exe = tmp_path / "client_cxx"
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-x", "c++", f"-I{ROOT / 'include'}",
                    str(ROOT / "tests" / "c_abi_client.c"), f"-L{PKG}", "-lpagedattn", f"-Wl,-rpath,{PKG}",
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout
    assert out.startswith("version ") and "unknown_sequence 1" in out


def test_status_and_version(client_output):
    from paged_kv_cache_331_b200 import _binding
    L = _binding.lib()
    assert int(client_output["version"][0]) == L.pa_version()
    names = {int(s): n for s, n in client_output["status"]}
    assert names == {s: L.pa_status_string(s).decode() for s in range(6)}


def test_argument_errors_before_any_launch(client_output):
    assert client_output["store_negative"] == ["1"]
    assert client_output["decode_head_dim_96"][0] == "2"         # PA_ERR_UNSUPPORTED, with a message
    assert "head_dim" in " ".join(client_output["decode_head_dim_96"][1:])


def test_xxh64_from_c(client_output):
    assert int(client_output["xxh64_empty"][0]) == xxhash.xxh64_intdigest(b"", seed=0)
    assert int(client_output["xxh64_abc"][0]) == xxhash.xxh64_intdigest(b"abc", seed=0)


def test_block_manager_from_c_matches_the_oracle(client_output):
    orc = OracleBlockManager(16, 4)
    orc.add_sequence(100, list(range(1, 11)))
    orc.add_sequence(200, [1, 2, 3, 4, 5, 6, 7, 8, 11])
    orc.allocate(100)
    orc.allocate(200)
    s = client_output["seq200"]
    assert [int(s[1]), int(s[3]), int(s[5]), int(s[7])] == [9, orc.seqs[200].num_cached_tokens,
                                                            len(orc.seqs[200].block_table), orc.num_free_blocks()]
    m = orc.prepare_prefill([100, 200], 4)
    p = client_output["prefill"]
    assert int(p[1]) == len(m["slot_mapping"])
    assert [int(x) for x in p[3:6]] == m["cu_seqlens_q"].tolist()
    assert [int(x) for x in p[7:10]] == m["cu_seqlens_k"].tolist()
    assert [int(x) for x in client_output["tables"]] == m["block_tables"].ravel().tolist()
    assert [int(x) for x in client_output["slots"]] == m["slot_mapping"].tolist()
    orc.append_token(100, 42)
    orc.may_append(100)
    d = orc.prepare_decode([100, 200], 4)
    got = [int(x) for x in client_output["decode"][1:3] + client_output["decode"][4:6] + client_output["decode"][7:9]]
    assert got == d["context_lens"].tolist() + d["slot_mapping"].tolist() + d["positions"].tolist()
    assert client_output["unknown_sequence"] == ["1"]
