"""GPU: the block pool driving the kernels -- prefix caching with forks and
copy-on-write (attn_copy_blocks), checked against the fp64 oracle."""

import math

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu

kv = pytest.importorskip("kv_cache_decode_attn_b200")
from tests.gpu_util import check_lse, check_o, f64, to_dev_i32  # noqa: E402


@pytest.fixture(autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    kv.attn_get_device_status(clear=True)
    yield
    assert kv.attn_get_device_status(clear=True) == 0


@pytest.mark.parametrize("prompt_len", [100, 96])
def test_prefix_caching_forks_with_copy_on_write(prompt_len):
    """One prompt written once; three completions fork from it, each appends its
    own tokens (the shared, partly filled last block is copied first) and
    attends over prompt + own tokens.  The prompt's blocks stay untouched."""
    Hq, Hkv, d, T, nblk, width = 8, 2, 128, 5, 64, 16
    pool = kv.BlockPool(nblk)
    k_pool = torch.zeros(nblk, 16, Hkv, d, dtype=torch.bfloat16, device="cuda")
    v_pool = torch.zeros_like(k_pool)
    pk = synth.normal_bf16((1, prompt_len, Hkv, d), 1, "cuda")
    pv = synth.normal_bf16((1, prompt_len, Hkv, d), 2, "cuda")
    root = pool.create()
    assert pool.reserve(root, prompt_len) == []
    table, _ = pool.page_table([root], width)
    kv.kv_append(k_pool, v_pool, pk, pv, to_dev_i32([0]), page_table=table.cuda())
    root_blocks = pool.blocks(root)
    snapshot = k_pool[root_blocks].clone(), v_pool[root_blocks].clone()

    children = [pool.fork(root) for _ in range(3)]
    copies = 0
    for i, c in enumerate(children):
        cow = pool.reserve(c, T)
        copies += len(cow)
        if cow:
            src = to_dev_i32([s for s, _ in cow])
            dst = to_dev_i32([t for _, t in cow])
            kv.copy_blocks(k_pool, v_pool, src, dst)
        kn = synth.normal_bf16((1, T, Hkv, d), 10 + i, "cuda")
        vn = synth.normal_bf16((1, T, Hkv, d), 20 + i, "cuda")
        q = synth.normal_bf16((1, T, Hq, d), 30 + i, "cuda")
        table, lens = pool.page_table([c], width)
        assert int(lens[0]) == prompt_len + T
        kv.kv_append(k_pool, v_pool, kn, vn, to_dev_i32([prompt_len]), page_table=table.cuda())
        o = torch.empty(1, T, Hq, d, device="cuda")
        lse = torch.empty(1, Hq, T, device="cuda")
        kv.attn_decode(q, k_pool, v_pool, lens.cuda(), o, lse, page_table=table.cuda())
        K = np.concatenate([f64(pk), f64(kn)], axis=1)
        V = np.concatenate([f64(pv), f64(vn)], axis=1)
        o_ref, lse_ref = oracle.decode(f64(q), K, V, [prompt_len + T], 1 / math.sqrt(d), True)
        check_o(o, o_ref, f"child {i}")
        check_lse(lse, lse_ref, f"child {i}")
    # a partly filled shared block is copied once per child; a full one never
    assert copies == (3 if prompt_len % 16 else 0)
    assert torch.equal(k_pool[root_blocks], snapshot[0]) and torch.equal(v_pool[root_blocks], snapshot[1])
    for c in children + [root]:
        pool.free(c)
    assert pool.free_blocks() == nblk


def test_copy_blocks_bit_exact_bf16_and_fp8():
    for dtype in (torch.bfloat16, torch.uint8):
        nblk, Hkv, d = 12, 4, 128
        g = torch.Generator(device="cuda").manual_seed(3)
        if dtype == torch.uint8:
            k = torch.randint(0, 256, (nblk, 16, Hkv, d), generator=g, device="cuda", dtype=torch.uint8)
        else:
            k = torch.randn(nblk, 16, Hkv, d, generator=g, device="cuda").to(dtype)
        v = k.flip(0).clone()
        k0, v0 = k.clone(), v.clone()
        src, dst = [1, 5, 9], [7, 2, 11]
        kv.copy_blocks(k, v, to_dev_i32(src), to_dev_i32(dst))
        for s, t in zip(src, dst):
            assert torch.equal(k[t], k0[s]) and torch.equal(v[t], v0[s])
        untouched = [i for i in range(nblk) if i not in dst]
        assert torch.equal(k[untouched], k0[untouched]) and torch.equal(v[untouched], v0[untouched])


def test_copy_blocks_bad_id_sets_status():
    k = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    v = torch.zeros_like(k)
    kv.copy_blocks(k, v, to_dev_i32([0, 9]), to_dev_i32([1, 2]))
    assert kv.attn_get_device_status(clear=True) & kv.ATTN_DEV_PAGE_ID
