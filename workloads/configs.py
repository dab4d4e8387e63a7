"""The five SANA-WM-shaped GDN workloads, as plain data.

Shapes follow the SANA-WM pages: the Stage-1 DiT has 20 heads of head_dim 112
(sglang cookbook, section 1 architecture table), a latent frame at 704x1280
with a 32x32 VAE stride is 22x40 = 880 tokens (same table, VAE and output
rows), streaming blocks hold 3 latent frames (sglang cookbook, section 9,
``num_frame_per_block``), a 241-frame clip is 31 latent frames (FlashDreams
runner page, profiling benchmark) and a minute at 16 fps is 121 latent frames
(sglang cookbook, section 1 output row; frame counts snap to 8k+1).

Nothing here computes any part of the method; it only names sizes and the
distributions the seeded generator in ``workloads.synth`` draws from.
"""

from dataclasses import dataclass, field, replace
from typing import Optional

TOKENS_PER_FRAME = 880          # 22 x 40 latent grid, patch 1
FRAMES_PER_BLOCK = 3            # streaming block
HEADS = 20
HEAD_DIM = 112


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d_k: int
    d_v: int
    frame_len: int
    chunk_len: int
    io_dtype: str                 # "bf16" or "f32": element type of q, k, v, out
    gate_mean: float              # gate logits ~ N(gate_mean, gate_std) per frame
    gate_std: float
    beta_mean: float = 0.0        # beta logits ~ N(beta_mean, beta_std) per token
    beta_std: float = 1.0
    state_std: Optional[float] = None   # None: zero initial state
    seed: int = 0
    layers: int = 1               # independent layers timed back-to-back
    blocks: int = 1               # successive streaming blocks (state carried)
    session_seed_base: Optional[int] = None   # per-session seeds (batched streaming)
    note: str = ""

    @property
    def n_frames(self) -> int:
        return -(-self.T // self.frame_len)

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


TINY = Workload(
    name="tiny", B=1, H=2, T=64, d_k=32, d_v=32, frame_len=16, chunk_len=16,
    io_dtype="f32", gate_mean=0.0, gate_std=1.0, state_std=None, seed=0,
    note="4 latent frames x 16 tokens, fp32 q/k/v, zero initial state")

BLOCK = Workload(
    name="block", B=1, H=HEADS, T=FRAMES_PER_BLOCK * TOKENS_PER_FRAME,
    d_k=HEAD_DIM, d_v=HEAD_DIM, frame_len=TOKENS_PER_FRAME, chunk_len=64,
    io_dtype="bf16", gate_mean=2.0, gate_std=0.5, state_std=0.02, seed=0,
    note="one streaming block (3 latent frames), state carried in and out")

CLIP241 = Workload(
    name="clip241", B=1, H=HEADS, T=31 * TOKENS_PER_FRAME,
    d_k=HEAD_DIM, d_v=HEAD_DIM, frame_len=TOKENS_PER_FRAME, chunk_len=64,
    io_dtype="bf16", gate_mean=2.0, gate_std=0.5, state_std=None, seed=0,
    note="241-frame clip = 31 latent frames, zero initial state")

MINUTE = Workload(
    name="minute", B=1, H=HEADS, T=121 * TOKENS_PER_FRAME,
    d_k=HEAD_DIM, d_v=HEAD_DIM, frame_len=TOKENS_PER_FRAME, chunk_len=64,
    io_dtype="bf16", gate_mean=2.0, gate_std=0.5, state_std=None, seed=0,
    layers=20,
    note="minute-scale layer = 121 latent frames (106,480 tokens); 20 layers back-to-back")

SESSIONS = Workload(
    name="sessions", B=4, H=HEADS, T=FRAMES_PER_BLOCK * TOKENS_PER_FRAME,
    d_k=HEAD_DIM, d_v=HEAD_DIM, frame_len=TOKENS_PER_FRAME, chunk_len=64,
    io_dtype="bf16", gate_mean=2.0, gate_std=0.5, state_std=0.02, seed=0,
    blocks=40, session_seed_base=1000,
    note="4 independent sessions x 40 successive 3-frame blocks, state carried block to block")

CONFIGS = {w.name: w for w in (TINY, BLOCK, CLIP241, MINUTE, SESSIONS)}


def long_memory(w: Workload) -> Workload:
    """Variant with slow decay (gate logits ~ N(-6, 0.5), a ~ 0.9975 per token).

    With the configs' N(2, 0.5) logits a token's gate is about 0.12, so the
    carried state is forgotten within a few dozen tokens; this variant keeps
    about 11 % of the state across a frame and exercises the long-range carry.
    """
    return w.with_(name=w.name + "_longmem", gate_mean=-6.0, gate_std=0.5,
                   state_std=0.02 if w.state_std is None else w.state_std)
