"""The whole step through h2o_chunk_step against the oracle: teacher-forced
and free-running trajectories on the workloads' generators, the host-buffer
entry point, checkpoint/resume, and a sampled check at full size."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.workloads import QWEN_C8K, TINY, ChunkSource, DeviceChunkSource
from oracle import h2o_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


def shape_for(wl, **over):
    dt = wl.torch_dtype()
    s = dict(B=wl.batch, Hq=wl.n_q_heads, Hkv=wl.n_kv_heads, d=wl.head_dim, C=wl.capacity,
             max_chunk=wl.chunk, W=wl.window, dtype=dt)
    s.update(over)
    return gh.shape_of(s["B"], s["Hq"], s["Hkv"], s["d"], s["C"], s["max_chunk"], s["W"],
                       s["dtype"])


def run_trajectory(wl, steps, teacher_forced, resync=True):
    """Runs `steps` chunks on both sides; returns the near-tie step count."""
    src = ChunkSource(wl, seed=0)
    shape = shape_for(wl)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    G = wl.group
    near_ties = 0
    for c in range(steps):
        q, kn, vn = src.chunk(c)
        if teacher_forced:
            gh.push_oracle_state(gpu, ref)
        O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
        O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
        gh.assert_attention_close(O, cs, O_ref, cs_ref, wl.chunk, G, f"{wl.name} step {c}")
        cs32 = cs_ref.astype(np.float32)
        gap = gh.min_gap(ref, cs32, wl.chunk)
        ref.evict(cs32, gh.np64(kn), gh.np64(vn))
        st = gpu.read()
        if gap > gh.GAP_RTOL:
            # identical kept sets; scores may differ in the last bits only
            # through the summed weights, so compare positions and contents
            assert np.array_equal(st["pos"].cpu().numpy(), ref.pos), f"step {c}: kept set"
            assert torch.equal(gh.bits(st["k"]), gh.bits(torch.from_numpy(ref.K).to(shape.dtype)))
            assert torch.equal(gh.bits(st["v"]), gh.bits(torch.from_numpy(ref.V).to(shape.dtype)))
            assert np.allclose(st["scores"].cpu().numpy(), ref.scores, rtol=2e-3, atol=1e-6)
        else:
            near_ties += 1
            if resync:
                gh.push_oracle_state(gpu, ref)
        assert st["n"] == ref.n and st["t0"] == ref.t0
    assert gpu.check() == 0
    return near_ties


def test_tiny_workload_teacher_forced():
    run_trajectory(TINY, TINY.steps, teacher_forced=True)


def test_tiny_workload_free_running():
    run_trajectory(TINY, TINY.steps, teacher_forced=False)


SMALL_QWEN = QWEN_C8K.scaled(name="qwen_small", n_q_heads=8, n_kv_heads=2, chunk=256,
                             capacity=1024, window=64, seq_len=256 * 7)


def test_scaled_qwen_free_running():
    """Qwen-shaped heads (d = 128, G = 4) at reduced sizes, 7 steps: fill,
    then eviction with a protected window."""
    run_trajectory(SMALL_QWEN, SMALL_QWEN.steps, teacher_forced=False)


def test_ragged_chunks_and_windows():
    for W, nq in ((0, 100), (100, 100), (150, 100), (0, 1)):
        wl = SMALL_QWEN.scaled(name=f"ragged_{W}_{nq}", chunk=nq, capacity=300, window=W,
                               seq_len=nq * 5)
        run_trajectory(wl, 5, teacher_forced=True)


def test_host_entry_point_matches_device_entry_point():
    wl = SMALL_QWEN
    src = ChunkSource(wl, seed=1)
    shape = shape_for(wl)
    a = binding.H2OCache(shape)
    b = binding.H2OCache(shape)
    for c in range(5):
        q, kn, vn = src.chunk(c)
        Oa = a.step(q.cuda(), kn.cuda(), vn.cuda())
        out = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        b.step_host(q.pin_memory(), kn.pin_memory(), vn.pin_memory(), out)
        torch.cuda.synchronize()
        assert torch.equal(gh.bits(Oa), gh.bits(out))
    sa, sb = a.read(), b.read()
    for key in ("k", "v", "scores", "pos"):
        assert torch.equal(gh.bits(sa[key]), gh.bits(sb[key])), key


def test_pipelined_host_steps_match_device_steps():
    """Several host-buffer steps in flight at once (no join between them, a
    side stream, chunk sizes that change between calls): after one join every
    output and the final cache equal the device-buffer path bit for bit."""
    wl = SMALL_QWEN.scaled(name="pipelined", capacity=300, window=40, chunk=100, seq_len=700)
    src = ChunkSource(wl, seed=3)
    shape = shape_for(wl)
    a = binding.H2OCache(shape)
    b = binding.H2OCache(shape)
    sizes = (100, 37, 100, 1, 64, 100, 99)
    chunks = [src.chunk(c, n_q=nq) for c, nq in enumerate(sizes)]
    ref = [a.step(*(t.cuda() for t in ch)) for ch in chunks]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    host_in = [tuple(t.pin_memory() for t in ch) for ch in chunks]
    outs = [torch.full(ch[0].shape, float("nan"), dtype=ch[0].dtype).pin_memory()
            for ch in chunks]
    with torch.cuda.stream(side):
        for (q, kn, vn), out in zip(host_in, outs):
            b.step_host(q, kn, vn, out, stream=side, join=False)
        b.host_join(side)
    side.synchronize()
    for r, out in zip(ref, outs):
        assert torch.equal(gh.bits(r), gh.bits(out))
    sa, sb = a.read(), b.read()
    for key in ("k", "v", "scores", "pos"):
        assert torch.equal(gh.bits(sa[key]), gh.bits(sb[key])), key


def test_checkpoint_resume_bit_exact():
    wl = SMALL_QWEN
    src = ChunkSource(wl, seed=2)
    chunks = [src.chunk(c) for c in range(7)]
    shape = shape_for(wl)
    a = binding.H2OCache(shape)
    for c in chunks[:5]:
        a.step(*(t.cuda() for t in c))
    snap = a.read()
    b = binding.H2OCache(shape)
    b.write(snap["k"], snap["v"], snap["scores"], snap["pos"], snap["n"], snap["t0"])
    for c in chunks[5:]:
        Oa, ca = a.step(*(t.cuda() for t in c), return_colsum=True)
        Ob, cb = b.step(*(t.cuda() for t in c), return_colsum=True)
        assert torch.equal(gh.bits(Oa), gh.bits(Ob)) and torch.equal(gh.bits(ca), gh.bits(cb))
    sa, sb = a.read(), b.read()
    for key in ("k", "v", "scores", "pos"):
        assert torch.equal(gh.bits(sa[key]), gh.bits(sb[key])), key
    assert (sa["n"], sa["t0"]) == (sb["n"], sb["t0"])


def test_launch_count_and_state_word():
    shape = shape_for(SMALL_QWEN)
    gpu = binding.H2OCache(shape)
    q, kn, vn = ChunkSource(SMALL_QWEN, seed=3).chunk(0)
    before = gpu.info()["kernel_launches"]
    gpu.step(q.cuda(), kn.cuda(), vn.cuda())
    assert gpu.info()["kernel_launches"] - before == 3
    assert gpu.check() == 0
    st = gpu.state.cpu().tolist()
    assert st[0] == 256 and st[1] == 256 and st[2] == 0


def test_full_size_qwen_sampled():
    """The Qwen3-4B-shaped workload (C = 8192, n_q = 1024, W = 256) at full
    size in the bench's launch configuration: fill the cache with device-drawn
    chunks, then one steady-state step checked against the oracle on two KV
    groups (8 heads) read back from the GPU, and the eviction checked
    bit-exactly when fed the GPU's own summed weights."""
    wl = QWEN_C8K
    shape = shape_for(wl)
    gpu = binding.H2OCache(shape)
    dev = torch.device("cuda")
    src = DeviceChunkSource(wl, 0, dev)
    for c in range(wl.capacity // wl.chunk + 1):
        gpu.step(*src.chunk(c))
    assert gpu.check() == 0
    st = gpu.read()
    assert st["n"] == wl.capacity
    q, kn, vn = src.chunk(wl.capacity // wl.chunk + 1)
    O, cs = gpu.attention(q, kn, vn)
    G = wl.group
    tot = gh.np64(cs).sum(-1)
    assert np.allclose(tot, wl.chunk * G, rtol=1e-4)
    # oracle on KV groups 0 and 5 (query heads 0..3 and 20..23)
    for g in (0, 5):
        heads = list(range(g * G, (g + 1) * G))
        o_ref, cs_ref, _ = orc.attention_one_cache(
            gh.np64(q[0, :, heads]), gh.np64(st["k"][0, g:g + 1]), gh.np64(st["v"][0, g:g + 1]),
            st["n"], gh.np64(kn[0, :, g:g + 1]), gh.np64(vn[0, :, g:g + 1]),
            1.0 / np.sqrt(wl.head_dim))
        gh.assert_attention_close(O[0, :, heads], cs[0, g:g + 1], o_ref, cs_ref, wl.chunk, G,
                                  f"group {g}")
    # eviction fed the GPU's own weights: bit-exact against the oracle
    ref = gh.oracle_for(shape)
    gh.load_oracle_from_gpu(ref, st)
    gpu.evict(cs, kn, vn)
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, shape.dtype, "full-size eviction")
    assert gpu.check() == 0
