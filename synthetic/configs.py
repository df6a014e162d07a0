"""The five synthetic workloads of the VDN hybrid layer.

Shapes follow the latent video token grid of "Video DeltaNet: A Video-Native
Hybrid Attention for Livestream Video Generation" (abstract; the sd114.wiki
article, section on the bidirectional sliding-window softmax branch: 5 latent
frames per block). The pages give no latent sizes, so each workload fixes
B (batch), H (heads), d (key/query dim), dv (value dim), T (latent frames)
and N (spatial tokens per frame). The 768p workload stands in for the pages'
768p, 14.4-second clip.
"""
from dataclasses import dataclass, field, replace


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    dv: int
    T: int
    N: int
    dtype: str            # "f32" or "bf16": element type of q, k, v, W and of every output
    lam: float            # ridge term lambda of the per-frame solve
    beta: float           # step size beta in (0, 1]
    seed: int
    block_frames: int = 5
    window_blocks: int = 1
    anchors: int = 1
    keys: str = "gauss"   # "gauss" | "student_t" | "rank_deficient"
    d_out: int = 0        # merge output width (0: no merge in this workload)
    w_per_head: int = 0   # 1: W1, W2 are dv x d_out and shared by all heads
    softmax: bool = True  # False: linear branch only (long-scan stress)
    grid: tuple = field(default=(0, 0))  # spatial grid (rows, cols), N = rows * cols
    extra: dict = field(default_factory=dict)
    n_ctx: int = 0        # context (text / audio) tokens after the T*N video tokens of a head

    @property
    def L(self) -> int:
        return self.T * self.N + self.n_ctx

    @property
    def nb(self) -> int:
        return -(-self.T // self.block_frames)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload(
        name="tiny", B=1, H=2, d=64, dv=64, T=20, N=64, grid=(8, 8), dtype="f32",
        lam=1e-3, beta=0.5, seed=0, d_out=64, w_per_head=1),
    "small": Workload(
        name="small", B=1, H=8, d=128, dv=128, T=40, N=1008, grid=(24, 42), dtype="bf16",
        lam=1e-2, beta=1.0, seed=1, d_out=1024),
    "768p": Workload(
        name="768p", B=1, H=24, d=128, dv=128, T=60, N=4032, grid=(48, 84), dtype="bf16",
        lam=1e-2, beta=0.8, seed=2, d_out=3072),
    "vda_only": Workload(
        name="vda_only", B=2, H=16, d=128, dv=128, T=240, N=1024, grid=(32, 32), dtype="bf16",
        lam=1e-3, beta=1.0, seed=3, keys="rank_deficient", softmax=False,
        extra={"deficient_frac": 0.1, "rank": 16}),
    "ragged": Workload(
        name="ragged", B=2, H=16, d=128, dv=128, T=61, N=2520, grid=(36, 70), dtype="bf16",
        lam=1e-2, beta=0.5, seed=4, keys="student_t", d_out=2048,
        extra={"nu": 3}),
}


def get_workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w
