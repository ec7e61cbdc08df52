"""The layer-by-layer decode of a stack into one reused scratch buffer, as
the decode-before-use pattern runs it: embedding, three Qwen3-8B-shaped
blocks and the LM head, one DecodePlan per layer on one stream with
programmatic dependent launch on.

Two orders are checked:
  - after each layer's decode, kernels that are not decodes read the
    scratch buffer (a checksum, and a copy out) before the next layer's
    decode overwrites it;
  - two layers' decodes back to back into the same buffer, with nothing in
    between: the second launch may start while the first finishes, and must
    still leave exactly its own words.
Every tensor is compared with the original (regenerated from its seed on the
device), and sampled format blocks with the CPU oracle's decode.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

df11 = pytest.importorskip("huffman_decode_df11_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()


def _groups(names):
    groups, cur, key = [], [], None
    for i, n in enumerate(names):
        k = n.split(".")[1] if n.startswith("layers.") else n
        if cur and k != key:
            groups.append(cur)
            cur = []
        key = k
        cur.append(i)
    groups.append(cur)
    return groups


def _sampled_blocks_vs_oracle(h, got_u16, samples=6):
    """Sampled format blocks decoded by the oracle from their first codeword."""
    p = h.params
    T, C = p.threads_per_block, p.chunk_bytes
    gaps = np.unpackbits(h.gaps)
    nb = p.num_blocks
    picks = sorted(set([0, nb - 1] + list(np.random.default_rng(1).integers(0, nb, samples))))
    for b in picks:
        c = b * T
        g = int("".join(str(int(x)) for x in gaps[5 * c:5 * c + 5]), 2)
        lo, hi = int(h.block_out_pos[b]), int(h.block_out_pos[b + 1])
        if hi == lo:
            continue
        ref, _, _ = oracle.decode(h.bitstream, h.code_lengths, h.sign_mantissa[lo:], hi - lo,
                                  start_bit=c * C * 8 + g)
        assert np.array_equal(got_u16[lo:hi], ref), b


@pytest.fixture(scope="module")
def stack():
    units = workloads.stack_units(seed=3, layers=3)
    names = [u[0] for u in units]
    groups = _groups(names)
    devs = [None] * len(units)
    for g in groups:
        ws = [units[i][2]("cuda") for i in g]
        for i, d in zip(g, df11.compress_on_device_batched(ws)):
            devs[i] = d
        del ws
    sizes = [sum(devs[i].n for i in g) for g in groups]
    scratch = torch.empty(max(sizes), dtype=torch.int16, device="cuda")
    outs = []
    for g in groups:
        off, o = 0, []
        for i in g:
            o.append(scratch[off:off + devs[i].n])
            off += devs[i].n
        outs.append(o)
    plans = [df11.DecodePlan([devs[i] for i in g], o) for g, o in zip(groups, outs)]
    return units, groups, devs, scratch, outs, plans


def test_layers_with_consumers_between_them(stack):
    units, groups, devs, scratch, outs, plans = stack
    assert len(groups) == 5 and [len(g) for g in groups] == [1, 7, 7, 7, 1]
    err = df11.new_error_word()
    sums = torch.zeros(len(groups), dtype=torch.int64, device="cuda")
    copies = [[torch.empty_like(o) for o in os_] for os_ in outs]
    for gi, plan in enumerate(plans):
        plan.run(err=err)
        n = sum(o.numel() for o in outs[gi])
        sums[gi] = scratch[:n].to(torch.int64).sum()       # reads the decoded weights
        for c, o in zip(copies[gi], outs[gi]):
            c.copy_(o)
    torch.cuda.synchronize()
    df11.check_device_error(err)
    for gi, g in enumerate(groups):
        total = 0
        for i, c in zip(g, copies[gi]):
            ref = units[i][2]("cuda")
            assert torch.equal(c, ref), units[i][0]
            total += int(ref.to(torch.int64).sum())
            del ref
        assert int(sums[gi]) == total, gi
    # the oracle on sampled blocks: the embedding, one block weight, the LM head
    for gi, k in ((0, 0), (2, 4), (4, 0)):
        h = df11.to_host(devs[groups[gi][k]])
        _sampled_blocks_vs_oracle(h, copies[gi][k].cpu().numpy().view(np.uint16))


def test_layer_decodes_back_to_back_into_one_buffer(stack):
    units, groups, devs, scratch, outs, plans = stack
    err = df11.new_error_word()
    for a in range(len(plans) - 1):
        scratch.fill_(-1)
        plans[a].run(err=err)
        plans[a + 1].run(err=err)  # overwrites what plans[a] wrote
        torch.cuda.synchronize()
        for i, o in zip(groups[a + 1], outs[a + 1]):
            assert torch.equal(o, units[i][2]("cuda")), (a, units[i][0])
    df11.check_device_error(err)
