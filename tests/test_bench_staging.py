"""Host-side staging of bench.py on CPU: the packed layouts that let one copy upload a
step's metadata (and, end to end, a layer's q and K / V rows), and one append launch write
the step's token rows and its admitted prompts' rows."""
import numpy as np
import pytest
import torch

import bench


N = 5


def _meta(n=N, mb=7, max_prompt=11):
    # the benchmark's layout: slots last, the n token slots then the prompt slots
    return bench.Packed([("tables", torch.int32, (n, mb)), ("lens", torch.int32, (n,)),
                         ("cow", torch.int32, (n, 2)), ("slots", torch.int64, (n + max_prompt,))])


def test_parts_are_aligned_disjoint_and_in_order():
    m = _meta()
    prev_end = 0
    for name, dt, shape, off, nbytes in m.parts:
        assert off % bench.Packed.ALIGN == 0 and off >= prev_end
        assert nbytes == int(np.prod(shape)) * dt.itemsize
        prev_end = off + nbytes
    assert m.nbytes >= prev_end and m.nbytes % bench.Packed.ALIGN == 0


def test_views_have_the_part_shapes_and_write_through():
    m = _meta()
    buf = torch.zeros(m.nbytes, dtype=torch.uint8)
    v = m.views(buf)
    assert v["tables"].shape == (5, 7) and v["tables"].dtype == torch.int32 and v["tables"].is_contiguous()
    assert v["cow"].shape == (5, 2) and v["slots"].dtype == torch.int64 and v["slots"].shape == (5 + 11,)
    v["tables"][:] = torch.arange(35, dtype=torch.int32).view(5, 7)
    v["slots"][N:N + 3] = torch.tensor([7, -1, 1 << 40])
    w = m.views(buf.clone())
    assert torch.equal(w["tables"], v["tables"]) and w["slots"][N:N + 3].tolist() == [7, -1, 1 << 40]


def test_token_and_prompt_slots_are_one_run():
    """The step reserves the prompts' slots into slots[n:] and the token slots into
    slots[:n]; the append launch then reads slots[:n + ptot] in the order of its rows."""
    m = _meta()
    v = m.views(torch.zeros(m.nbytes, dtype=torch.uint8))
    tok, prm = v["slots"][:N], v["slots"][N:]
    tok.copy_(torch.arange(100, 100 + N))
    prm[:4].copy_(torch.tensor([3, 4, 5, 6]))
    assert v["slots"][:N + 4].tolist() == list(range(100, 100 + N)) + [3, 4, 5, 6]
    assert tok.data_ptr() + N * 8 == prm.data_ptr()


def test_one_prefix_copy_carries_every_part_and_the_used_prompt_slots():
    m = _meta()
    host = torch.zeros(m.nbytes, dtype=torch.uint8)
    hv = m.views(host)
    rng = np.random.default_rng(0)
    for name in ("tables", "lens", "cow", "slots"):
        hv[name].copy_(torch.from_numpy(rng.integers(-9, 1 << 20, hv[name].shape).astype(
            np.int64 if hv[name].dtype == torch.int64 else np.int32)))
    ptot = 4
    nb = m.off["slots"] + (N + ptot) * 8
    dev = torch.full((m.nbytes,), 0xEE, dtype=torch.uint8)
    dev[:nb].copy_(host[:nb])
    dv = m.views(dev)
    for name in ("tables", "lens", "cow"):
        assert torch.equal(dv[name], hv[name])
    assert torch.equal(dv["slots"][:N + ptot], hv["slots"][:N + ptot])
    assert not torch.equal(dv["slots"][N + ptot:], hv["slots"][N + ptot:])   # unused slots were not copied


def test_empty_part():
    p = bench.Packed([("q", torch.bfloat16, (4, 2, 8)), ("a", torch.bfloat16, (0, 2, 8)),
                      ("b", torch.bfloat16, (0, 2, 8))])
    v = p.views(torch.zeros(p.nbytes, dtype=torch.uint8))
    assert v["a"].shape == (0, 2, 8) and v["b"].numel() == 0
    assert p.end["q"] == 4 * 2 * 8 * 2 and p.off["a"] == bench.Packed.ALIGN
    assert p.end["b"] == p.off["b"] == p.off["a"]


@pytest.mark.parametrize("workload", ["large_pool_b16", "large_pool_b32", "prefix_sharing", "worked_example"])
def test_fixed_batch_pools_hold_every_step_of_a_run(workload):
    """A fixed batch grows by one token per sequence and step; the benchmark's default run
    (warm-up, every timed pass, the end-to-end passes) must fit its pool."""
    import bench
    a = bench.parse(["--workload", workload])
    total = a.warmup + a.repeats * a.steps + min(a.repeats, 3) * a.steps
    r = bench.make_recipe(workload, 0, total)
    sh = r["shape"]
    B = sh.block_size
    if workload == "prefix_sharing":
        shared = r["prefix"] // B
        need = shared + sum(-(-(r["prefix"] + int(x) + total) // B) - shared for x in r["suffix"])
    else:
        need = sum(-(-(int(L) + total) // B) for L in r["lens"])
    assert need <= sh.num_blocks, (need, sh.num_blocks)
