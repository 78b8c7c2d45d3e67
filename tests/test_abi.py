"""The C-ABI library loads without a GPU, exports every function the header
declares, and rejects bad arguments on the host before launching anything.
CPU only: every call here returns during host-side validation."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spx.h")


def declared_functions():
    src = open(HEADER, encoding="utf-8").read()
    return re.findall(r"SPX_API\s+[\w\s\*]+?\b(spx_\w+)\s*\(", src)


@pytest.fixture(scope="module")
def spx():
    from conftest import build_lib
    build_lib()
    import long_context_decode_indexpool_b200 as m
    return m


def test_header_declares_the_calls():
    names = declared_functions()
    for required in ("spx_pool_append", "spx_index_score", "spx_topk_blocks",
                     "spx_sparse_mla_attn", "spx_decode_fused", "spx_prefill_chunk"):
        assert required in names


def test_every_declared_symbol_is_exported(spx):
    out = subprocess.run(["nm", "-D", "--defined-only", spx.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (\w+)$", out, flags=re.M))
    declared = set(declared_functions())
    assert declared <= exported, declared - exported
    assert set(spx.EXPORTED) == declared
    lib = ctypes.CDLL(spx.LIB_PATH)
    for name in declared:
        assert getattr(lib, name) is not None


def test_status_strings_and_version(spx):
    assert spx.status_string(0) == "SPX_OK"
    for code, name in spx.STATUS.items():
        assert spx.status_string(code) == name
    assert spx.status_string(99) == "SPX_ERR_UNKNOWN"
    assert "sm_100a" in spx.version()


def test_dims_validation(spx):
    d = spx.dims(64, 1.0)
    assert (d.idx_heads, d.idx_dim, d.pool, d.topk_blocks, d.latent) == (32, 128, 4, 512, 512)
    for bad_heads in (0, 8, 24, 144):
        with pytest.raises(spx.SpxError) as e:
            spx.dims(bad_heads, 1.0)
        assert e.value.status == 3
    for bad_scale in (0.0, -1.0, float("nan"), float("inf")):
        with pytest.raises(spx.SpxError) as e:
            spx.dims(16, bad_scale)
        assert e.value.status == 1
    d = spx.dims(16, 1.0)
    d.idx_dim = 64
    with pytest.raises(spx.SpxError) as e:
        spx.spx_topk_workspace_size(d, 4, 1000)
    assert e.value.status == 3


FAKE = 1 << 20  # a 16-byte aligned non-null address; never dereferenced


def test_host_validation_rejects_before_launch(spx):
    d = spx.dims(64, 1.0)
    s = 0  # legacy stream handle: nothing is launched on these paths
    # pool weights must sum to one
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append(d, 1, FAKE, 1, [0.5, 0.5, 0.5, 0.0], FAKE, FAKE, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    # max_len beyond the pooled-cache capacity
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append(d, 1, FAKE, 1, [0.25] * 4, FAKE, FAKE, 16, FAKE, 65, stream=s)
    assert e.value.status == 2
    # null tail
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append(d, 1, FAKE, 1, [0.25] * 4, None, FAKE, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    # misaligned cache pointer
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append(d, 1, FAKE, 1, [0.25] * 4, FAKE, FAKE + 2, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    # score stride too small
    with pytest.raises(spx.SpxError) as e:
        spx.spx_index_score(d, 2, FAKE, FAKE, FAKE, 1024, FAKE, 4096, FAKE, 1000, stream=s)
    assert e.value.status == 2
    # workspace too small
    need = spx.spx_topk_workspace_size(d, 4, 1 << 20)
    assert need > 0
    with pytest.raises(spx.SpxError) as e:
        spx.spx_topk_blocks(d, 4, FAKE, 1 << 18, FAKE, 1 << 20, FAKE, FAKE, FAKE, need - 1, stream=s)
    assert e.value.status == 4
    # fused decode: latent capacity below max_len
    need = spx.spx_decode_workspace_size(d, 4, 8192)
    with pytest.raises(spx.SpxError) as e:
        spx.spx_decode_fused(d, 4, FAKE, [0.25] * 4, FAKE, FAKE, 2048, FAKE, FAKE, FAKE, FAKE,
                             FAKE, 4096, 8192, FAKE, ws=FAKE, ws_bytes=need, stream=s)
    assert e.value.status == 2
    with pytest.raises(spx.SpxError) as e:
        spx.spx_decode_fused(d, 4, FAKE, [0.25] * 4, FAKE, FAKE, 2048, FAKE, FAKE, FAKE, FAKE,
                             FAKE, 8192, 8192, FAKE, ws=FAKE, ws_bytes=need - 256, stream=s)
    assert e.value.status == 4
    # fused decode beyond 16M tokens per sequence: unsupported (512 selection chunks)
    big = (1 << 24) + 4
    with pytest.raises(spx.SpxError) as e:
        spx.spx_decode_fused(d, 1, FAKE, [0.25] * 4, FAKE, FAKE, big // 4, FAKE, FAKE, FAKE, FAKE,
                             FAKE, big, big, FAKE, ws=FAKE, ws_bytes=1 << 40, stream=s)
    assert e.value.status == 3
    # prefill beyond the caches
    with pytest.raises(spx.SpxError) as e:
        spx.spx_prefill_chunk(d, 64, FAKE, [0.25] * 4, FAKE, FAKE, 16, 10, FAKE, FAKE, FAKE, FAKE,
                              1 << 20, FAKE, ws=FAKE, ws_bytes=1 << 30, stream=s)
    assert e.value.status == 2


def test_workspace_sizes_scale(spx):
    d = spx.dims(64, 1.0)
    small = spx.spx_decode_workspace_size(d, 4, 8192)
    big = spx.spx_decode_workspace_size(d, 4, 1 << 20)
    assert 0 < small < big
    # 1M context, 4 sequences: scores (4 MiB) dominate, top-k lists are 512 KiB
    assert big < 64 << 20
    assert spx.spx_topk_workspace_size(d, 4, 2048) == 0  # one level, no scratch
    assert spx.spx_prefill_workspace_size(d, 4096, 131072) > 4096 * (135168 // 4) * 4


def test_int8_cache_host_validation(spx):
    d = spx.dims(64, 1.0)
    s = 0
    # the scale array is required and must be 4-byte aligned
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append_i8(d, 1, FAKE, 1, [0.25] * 4, FAKE, FAKE, None, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append_i8(d, 1, FAKE, 1, [0.25] * 4, FAKE, FAKE, FAKE + 2, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    # the bf16 checks apply too (weights summing to one, capacity)
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append_i8(d, 1, FAKE, 1, [0.5] * 4, FAKE, FAKE, FAKE, 16, FAKE, 8, stream=s)
    assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_pool_append_i8(d, 1, FAKE, 1, [0.25] * 4, FAKE, FAKE, FAKE, 16, FAKE, 65, stream=s)
    assert e.value.status == 2
    # scoring: workspace holds the query codes and folded head weights
    need = spx.spx_index_score_i8_workspace_size(d, 4)
    assert need >= 4 * 32 * 128 + 4 * 32 * 4
    assert spx.spx_index_score_i8_workspace_size(d, 8) > need
    with pytest.raises(spx.SpxError) as e:
        spx.spx_index_score_i8(d, 4, FAKE, FAKE, FAKE, FAKE, 1024, FAKE, 4096, FAKE, 1024, FAKE,
                               ws_bytes=need - 1, stream=s)
    assert e.value.status == 4
    with pytest.raises(spx.SpxError) as e:
        spx.spx_index_score_i8(d, 4, FAKE, FAKE, FAKE, None, 1024, FAKE, 4096, FAKE, 1024, FAKE,
                               ws_bytes=need, stream=s)
    assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_index_score_i8(d, 4, FAKE, FAKE, FAKE, FAKE, 1024, FAKE, 4096, FAKE, 1000, FAKE,
                               ws_bytes=need, stream=s)
    assert e.value.status == 2
    # INT8 prefill: scales required and 4-byte aligned, the bf16 prefill workspace
    need = spx.spx_prefill_workspace_size(d, 64, 10)
    for ks, status in ((None, 1), (FAKE + 2, 1)):
        with pytest.raises(spx.SpxError) as e:
            spx.spx_prefill_chunk_i8(d, 64, FAKE, [0.25] * 4, FAKE, FAKE, ks, 32, 10, FAKE, FAKE,
                                     FAKE, FAKE, 128, FAKE, ws=FAKE, ws_bytes=need, stream=s)
        assert e.value.status == status
    with pytest.raises(spx.SpxError) as e:
        spx.spx_prefill_chunk_i8(d, 64, FAKE, [0.25] * 4, FAKE, FAKE, FAKE, 32, 10, FAKE, FAKE,
                                 FAKE, FAKE, 128, FAKE, ws=FAKE, ws_bytes=need - 1, stream=s)
    assert e.value.status == 4
    # fused decode: same workspace as the bf16 call; scales required
    need = spx.spx_decode_workspace_size(d, 4, 8192)
    with pytest.raises(spx.SpxError) as e:
        spx.spx_decode_fused_i8(d, 4, FAKE, [0.25] * 4, FAKE, FAKE, None, 2048, FAKE, FAKE, FAKE,
                                FAKE, FAKE, 8192, 8192, FAKE, ws=FAKE, ws_bytes=need, stream=s)
    assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_decode_fused_i8(d, 4, FAKE, [0.25] * 4, FAKE, FAKE, FAKE, 2048, FAKE, FAKE, FAKE,
                                FAKE, FAKE, 8192, 8192, FAKE, ws=FAKE, ws_bytes=need - 256,
                                stream=s)
    assert e.value.status == 4


def test_selftest_host_validation(spx):
    s = 0
    for bad in (0, 999, 1_000_000_001):  # limit outside 1 us .. 1 s
        with pytest.raises(spx.SpxError) as e:
            spx.spx_selftest_wait_timeout(bad, FAKE, stream=s)
        assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_selftest_wait_timeout(1_000_000, None, stream=s)
    assert e.value.status == 1
    with pytest.raises(spx.SpxError) as e:
        spx.spx_selftest_wait_timeout(1_000_000, FAKE + 2, stream=s)
    assert e.value.status == 1
