"""Model shapes of the looped nGPT (Dory1.0-4B and a tiny stand-in).

A *block* is one attention sublayer followed by one MLP sublayer.  The
72-"layer" count of the Dory pages counts sublayers: 27 sliding-window and
9 full attention sublayers plus 36 MLP sublayers (paperlayer summary, §2
Architecture), i.e. 36 blocks split 8 input / 20 recurrent / 8 output
(HF model-card digest, architecture section).

``layer_types`` marks each physical block 0 = sliding-window (SWA) or
1 = full attention.  Within each of the three groups the pattern
SWA, SWA, SWA, full repeats by the block's index inside the group
(config.json ``layer_types`` as described on the MXFP8 explainer page,
hybrid-attention section).
"""
from dataclasses import dataclass, field


@dataclass(frozen=True)
class ModelShape:
    name: str
    d: int                 # hidden size
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int               # SwiGLU inner width F
    vocab: int
    n_in: int              # input blocks
    n_rec: int             # recurrent blocks (shared across loops)
    n_out: int             # output blocks
    swa_window: int
    rope_theta_swa: float = 1.0e4
    rope_theta_full: float = 1.0e7
    layer_types: tuple = field(default=None)

    def __post_init__(self):
        if self.layer_types is None:
            lt = []
            for n in (self.n_in, self.n_rec, self.n_out):
                lt += [1 if (i % 4) == 3 else 0 for i in range(n)]
            object.__setattr__(self, "layer_types", tuple(lt))
        assert len(self.layer_types) == self.n_blocks

    @property
    def n_blocks(self):
        return self.n_in + self.n_rec + self.n_out

    @property
    def qdim(self):
        return self.n_q_heads * self.head_dim

    @property
    def kvdim(self):
        return self.n_kv_heads * self.head_dim

    @property
    def qkvg_rows(self):
        # q rows, k rows, v rows, gate rows (one gate per q-head channel)
        return 2 * self.qdim + 2 * self.kvdim

    def block_groups(self):
        """(input, recurrent, output) lists of physical block indices."""
        a, b = self.n_in, self.n_in + self.n_rec
        return (list(range(0, a)), list(range(a, b)),
                list(range(b, self.n_blocks)))

    def params_per_block(self):
        d, F = self.d, self.ffn
        return self.qkvg_rows * d + d * self.qdim + 2 * F * d + d * F


TINY = ModelShape(name="tiny", d=256, n_q_heads=4, n_kv_heads=1, head_dim=64,
                  ffn=768, vocab=1024, n_in=2, n_rec=4, n_out=2,
                  swa_window=16)

DORY = ModelShape(name="dory-4b", d=2560, n_q_heads=16, n_kv_heads=4,
                  head_dim=160, ffn=10240, vocab=131072, n_in=8, n_rec=20,
                  n_out=8, swa_window=1024)


def tiny_with_blocks(n_in, n_rec, n_out, **kw):
    """Tiny widths with another block split (used for depth-count checks)."""
    base = dict(name=f"tiny-{n_in}-{n_rec}-{n_out}", d=64, n_q_heads=4,
                n_kv_heads=2, head_dim=16, ffn=96, vocab=128, n_in=n_in,
                n_rec=n_rec, n_out=n_out, swa_window=8)
    base.update(kw)
    return ModelShape(**base)


def dory_with_blocks(n_in, n_rec, n_out):
    """Dory widths (every kernel shape unchanged) with fewer blocks: a small
    case for profilers that must keep the device footprint to a few GB."""
    return ModelShape(name=f"dory-{n_in}-{n_rec}-{n_out}", d=2560,
                      n_q_heads=16, n_kv_heads=4, head_dim=160, ffn=10240,
                      vocab=131072, n_in=n_in, n_rec=n_rec, n_out=n_out,
                      swa_window=1024)
