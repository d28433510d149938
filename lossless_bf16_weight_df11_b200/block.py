"""A transformer block held in DF11 form and decoded right before its forward.

[Block] of the method's page: the weights of a whole transformer block are
decompressed together, in one batch, just before the block runs, and the BF16
copies are dropped after it.  DF11Block does that for a Llama-style decoder
block (q, o, k, v, gate, up, down; GQA attention, SwiGLU MLP, RMSNorm without
learned scales, no rotary embedding): forward() decodes the seven matrices
with one df11_decode_block_batch launch into a BF16 scratch buffer, runs the
block with PyTorch (cuBLAS matmuls, scaled-dot-product attention) and releases
the buffer, unless the caller passes one to reuse.  The decoded weights are
bit-identical to the originals, so the forward equals, bit for bit, the same
forward on resident BF16 weights (forward_reference).

The same page compresses the embedding table and the LM head too, but does not
batch them with a block: DF11Embedding and DF11LMHead each hold one matrix in
DF11 form and decode it with one df11_decode launch right before their lookup
or projection, dropping the BF16 copy after it.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.nn.functional as F

from . import codec

NAMES = ("q", "o", "k", "v", "gate", "up", "down")


@dataclass
class BlockShape:
    hidden: int
    heads: int
    kv_heads: int
    ffn: int

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads

    def matrix_shapes(self) -> dict[str, tuple[int, int]]:
        """(out, in) of each matrix."""
        h, kv, f = self.hidden, self.kv_heads * self.head_dim, self.ffn
        return {"q": (h, h), "o": (h, h), "k": (kv, h), "v": (kv, h),
                "gate": (f, h), "up": (f, h), "down": (h, f)}


def _rms_norm(x: torch.Tensor, eps: float = 1e-5) -> torch.Tensor:
    xf = x.float()
    return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + eps)).to(x.dtype)


def block_forward(x: torch.Tensor, w: dict[str, torch.Tensor], shape: BlockShape) -> torch.Tensor:
    """One Llama-style block on BF16 activations x of shape (batch, seq, hidden)
    with BF16 weights w[name] of shape (out, in); causal attention."""
    b, s, h = x.shape
    hd = shape.head_dim
    a = _rms_norm(x)
    q = F.linear(a, w["q"]).view(b, s, shape.heads, hd).transpose(1, 2)
    k = F.linear(a, w["k"]).view(b, s, shape.kv_heads, hd).transpose(1, 2)
    v = F.linear(a, w["v"]).view(b, s, shape.kv_heads, hd).transpose(1, 2)
    rep = shape.heads // shape.kv_heads
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    att = F.scaled_dot_product_attention(q, k, v, is_causal=True)
    x = x + F.linear(att.transpose(1, 2).reshape(b, s, h), w["o"])
    m = _rms_norm(x)
    return x + F.linear(F.silu(F.linear(m, w["gate"])) * F.linear(m, w["up"]), w["down"])


class DF11Block:
    """The seven matrices of a block in DF11 form (one codebook each)."""

    def __init__(self, mats: dict[str, codec.DF11Matrix], shape: BlockShape):
        shapes = shape.matrix_shapes()
        for name in NAMES:
            if tuple(mats[name].shape) != shapes[name]:
                raise ValueError(f"{name}: shape {tuple(mats[name].shape)}, expected {shapes[name]}")
        self.mats = mats
        self.shape = shape

    @classmethod
    def compress(cls, weights: dict[str, torch.Tensor], shape: BlockShape,
                 cap: int = codec.DEFAULT_CAP) -> "DF11Block":
        mats = codec.compress_block([weights[n] for n in NAMES], cap=cap)
        return cls(dict(zip(NAMES, mats)), shape)

    @property
    def stored_bytes(self) -> int:
        return sum(m.stored_bytes for m in self.mats.values())

    def _offsets(self) -> tuple[dict[str, int], int]:
        # each matrix starts on a 16-byte boundary (8 BF16 values)
        offs, off = {}, 0
        for name in NAMES:
            offs[name] = off
            off += (self.mats[name].n + 7) // 8 * 8
        return offs, off

    def new_arena(self) -> torch.Tensor:
        """A BF16 scratch buffer large enough for the decoded block."""
        dev = self.mats["q"].stream.device
        return torch.empty(self._offsets()[1], dtype=torch.bfloat16, device=dev)

    def decode(self, arena: torch.Tensor | None = None, stream=None) -> dict[str, torch.Tensor]:
        """All seven matrices decoded by one launch into views of the arena."""
        offs, total = self._offsets()
        if arena is None:
            arena = self.new_arena()
        if arena.dtype != torch.bfloat16 or arena.numel() < total or arena.data_ptr() % 16:
            raise ValueError("arena: a 16-byte aligned BF16 buffer of at least new_arena()'s size")
        views = {}
        for name in NAMES:
            m = self.mats[name]
            views[name] = arena[offs[name]:offs[name] + m.n].view(m.shape)
        codec.decompress_block([self.mats[n] for n in NAMES], [views[n] for n in NAMES],
                               stream=stream)
        return views

    def forward(self, x: torch.Tensor, arena: torch.Tensor | None = None) -> torch.Tensor:
        """Decode the block, run it, drop the decoded weights (the arena is
        released here unless the caller owns it)."""
        w = self.decode(arena)
        y = block_forward(x, w, self.shape)
        del w
        return y

    def forward_reference(self, x: torch.Tensor, weights: dict[str, torch.Tensor]) -> torch.Tensor:
        """The same forward on resident BF16 weights."""
        return block_forward(x, weights, self.shape)


class _DF11Single:
    """One matrix in DF11 form, decoded by one df11_decode launch on use."""

    def __init__(self, mat: codec.DF11Matrix):
        if len(mat.shape) != 2:
            raise ValueError(f"expected a 2-D matrix, got shape {tuple(mat.shape)}")
        self.mat = mat

    @classmethod
    def compress(cls, weight: torch.Tensor, cap: int = codec.DEFAULT_CAP):
        if weight.dim() != 2 or weight.dtype != torch.bfloat16:
            raise ValueError("expected a 2-D BF16 weight")
        return cls(codec.compress(weight, cap=cap))

    @property
    def stored_bytes(self) -> int:
        return self.mat.stored_bytes

    def decode(self, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """The BF16 matrix (into out when given: a BF16 tensor of its shape)."""
        return codec.decompress(self.mat, out=out, stream=stream)


class DF11Embedding(_DF11Single):
    """A (vocab, hidden) embedding table in DF11 form."""

    def forward(self, ids: torch.Tensor, scratch: torch.Tensor | None = None) -> torch.Tensor:
        """Rows of the table for the token ids: the table is decoded, the rows
        gathered, and the decoded table dropped (unless it is the caller's
        scratch)."""
        w = self.decode(scratch)
        y = F.embedding(ids, w)
        del w
        return y

    def forward_reference(self, ids: torch.Tensor, weight: torch.Tensor) -> torch.Tensor:
        return F.embedding(ids, weight)


class DF11LMHead(_DF11Single):
    """A (vocab, hidden) output projection in DF11 form."""

    def forward(self, x: torch.Tensor, scratch: torch.Tensor | None = None) -> torch.Tensor:
        """Logits x W^T: W is decoded, used, and dropped (unless it is the
        caller's scratch)."""
        w = self.decode(scratch)
        y = F.linear(x, w)
        del w
        return y

    def forward_reference(self, x: torch.Tensor, weight: torch.Tensor) -> torch.Tensor:
        return F.linear(x, weight)
