"""DF11Block: a transformer block held in DF11 form, decoded by one launch right
before its forward.  The decoded weights are bit-identical to the originals, so
the block's output must equal, bit for bit, the same forward on the resident
BF16 weights (the same PyTorch operations on identical operands)."""
import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blockmod():
    from lossless_bf16_weight_df11_b200 import build
    build.build()
    import lossless_bf16_weight_df11_b200.block as b
    return b


def weights_for(shape, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = {}
    for name, (o, i) in shape.matrix_shapes().items():
        out[name] = (torch.randn(o, i, generator=g, device="cuda") / i ** 0.5).to(torch.bfloat16)
    return out


@pytest.mark.parametrize("tokens", [1, 16])
def test_small_block_matches_resident_forward(blockmod, tokens):
    shape = blockmod.BlockShape(hidden=512, heads=8, kv_heads=2, ffn=1536)
    w = weights_for(shape, seed=1)
    blk = blockmod.DF11Block.compress(w, shape)
    x = torch.randn(2, tokens, 512, device="cuda").to(torch.bfloat16)
    y = blk.forward(x)
    y_ref = blk.forward_reference(x, w)
    assert torch.equal(y, y_ref)
    assert blk.stored_bytes < 0.8 * sum(t.numel() * 2 for t in w.values())


def test_llama3_8b_block_with_reused_arena(blockmod):
    shape = blockmod.BlockShape(hidden=4096, heads=32, kv_heads=8, ffn=14336)
    names = [nm for nm, _ in workloads.WORKLOADS[3][1]]
    w = {nm: torch.from_numpy(workloads.matrix(3, i).view(np.int16)).cuda().view(torch.bfloat16)
         .reshape(shape.matrix_shapes()[nm]) for i, nm in enumerate(names)}
    blk = blockmod.DF11Block.compress(w, shape)
    arena = blk.new_arena()
    x = torch.randn(1, 8, 4096, device="cuda").to(torch.bfloat16)
    for _ in range(2):  # the arena is reused; the second decode overwrites the first
        y = blk.forward(x, arena=arena)
        assert torch.equal(y, blk.forward_reference(x, w))
    dec = blk.decode(arena)
    for nm in names:
        assert torch.equal(dec[nm].view(torch.int16), w[nm].view(torch.int16))


def test_shape_mismatch_rejected(blockmod):
    shape = blockmod.BlockShape(hidden=512, heads=8, kv_heads=2, ffn=1536)
    w = weights_for(shape, seed=2)
    blk = blockmod.DF11Block.compress(w, shape)
    with pytest.raises(ValueError):
        blockmod.DF11Block(blk.mats, blockmod.BlockShape(hidden=512, heads=8, kv_heads=4, ffn=1536))


@pytest.mark.parametrize("vocab,hidden", [(1000, 512), (32768, 1024)])
def test_embedding_and_lm_head_match_resident(blockmod, vocab, hidden):
    """The embedding lookup and the LM-head projection on a table held in
    DF11 form equal, bit for bit, the same operations on the resident table;
    a caller-owned scratch buffer gives the same result."""
    g = torch.Generator(device="cuda")
    g.manual_seed(vocab)
    w = (torch.randn(vocab, hidden, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    emb = blockmod.DF11Embedding.compress(w)
    head = blockmod.DF11LMHead(emb.mat)
    ids = torch.randint(0, vocab, (3, 17), generator=g, device="cuda")
    assert torch.equal(emb.forward(ids), emb.forward_reference(ids, w))
    x = torch.randn(3, 17, hidden, generator=g, device="cuda").to(torch.bfloat16)
    assert torch.equal(head.forward(x), head.forward_reference(x, w))
    scratch = torch.empty(vocab, hidden, dtype=torch.bfloat16, device="cuda")
    assert torch.equal(head.forward(x, scratch=scratch), head.forward_reference(x, w))
    assert torch.equal(scratch.view(torch.int16), w.view(torch.int16))
    assert emb.stored_bytes < 0.8 * w.numel() * 2
    with pytest.raises(ValueError):
        blockmod.DF11Embedding.compress(w.reshape(-1))
