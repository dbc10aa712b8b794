"""Workload definitions and the synthetic input recipe.

Sizes follow the GLM-5.2 MoE layer described on the colibri pages (README
"思路": 256 routed experts per MoE layer, about 19 MB per expert in int4; README
"已实现的功能": DeepSeek-V3-like sigmoid router with a shared expert), plus a
tiny layer the CPU oracle finishes in seconds.  No arithmetic of the layer is
done here: the module names shapes, seeds and distributions only.

Input recipe (every array is a pure function of (seed, stream, index); see
``synth``):
  - expert weights gate/up [I][H] and down [H][I]: f32 N(0, 0.02), quantised
    per row to the configured format by the layer's own quantiser;
  - router weight Wr [E][H]: f32 N(0, 0.02);
  - score-correction bias [E]: f32 N(0, bias_std);
  - activations x [T][H]: N(0, 1), f32 or bf16;
  - weights and router: drawn from the layer seed -- 1000 for the tiny layer,
    1001 for the GLM-shaped layer, which every GLM-shaped workload shares (the
    decode, verify/prefill and format-sweep workloads all run "the same
    GLM-shaped layer");
  - bias and activations: drawn from the workload seed 1000 + workload id;
    batch b of a workload draws x from stream (X, b), so a benchmark can
    rotate through distinct batches.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

A_F32, A_Q8, A_BF16 = 0, 1, 2
AFMT_NAMES = {A_F32: "f32", A_Q8: "q8_0", A_BF16: "bf16"}

# stream ids: (kind << 32) | index
K_GATE, K_UP, K_DOWN, K_WR, K_BIAS, K_X, K_XC = 1, 2, 3, 4, 5, 6, 7
W_STD = 0.02


def stream(kind: int, index: int = 0) -> int:
    return (kind << 32) | index


@dataclass(frozen=True)
class Workload:
    name: str
    wid: int                   # workload id (seed = 1000 + wid)
    hidden: int
    n_experts: int
    inter: int
    n_group: int
    topk_group: int
    top_k: int
    rsf: float
    wbits: int
    afmt: int
    T: int
    bias_std: float

    @property
    def seed(self) -> int:
        """Seed of the bias and the activations."""
        return 1000 + self.wid

    @property
    def layer_seed(self) -> int:
        """Seed of the expert weights and the router weight."""
        return 1000 if self.hidden == 256 else 1001

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    def expert_bytes(self, wbits: int | None = None) -> int:
        """Packed bytes of one expert (gate, up, down) plus its f32 row scales."""
        b = self.wbits if wbits is None else wbits
        H, I = self.hidden, self.inter
        return 3 * H * I * b // 8 + (2 * I + H) * 4


TINY = Workload("tiny_t8_int4_f32", 0, 256, 16, 128, 4, 2, 4, 2.5, 4, A_F32, 8, 0.1)
GLM = dict(hidden=6144, n_experts=256, inter=2048, n_group=8, topk_group=4, top_k=8, rsf=2.5)
GLM_DECODE_T1 = Workload("glm_decode_t1_int4_f32", 1, **GLM, wbits=4, afmt=A_F32, T=1,
                         bias_std=0.1)
GLM_DECODE_T32_Q8 = Workload("glm_decode_t32_int4_q8", 2, **GLM, wbits=4, afmt=A_Q8, T=32,
                             bias_std=0.5)
GLM_VERIFY_T4_BF16 = Workload("glm_verify_t4_int4_bf16", 3, **GLM, wbits=4, afmt=A_BF16, T=4,
                              bias_std=0.1)
GLM_PREFILL_T2048_BF16 = GLM_VERIFY_T4_BF16.with_(name="glm_prefill_t2048_int4_bf16", T=2048)


def sweep() -> list[Workload]:
    """Format sweep on the GLM-shaped layer: {int8, int4, int2} x {f32, Q8_0} x T in {1, 64}."""
    out = []
    for wb in (8, 4, 2):
        for af in (A_F32, A_Q8):
            for T in (1, 64):
                out.append(Workload(f"glm_sweep_int{wb}_{AFMT_NAMES[af]}_t{T}", 4, **GLM,
                                    wbits=wb, afmt=af, T=T, bias_std=0.1))
    return out


# Smallest layer the tensor-core expert engine takes (bf16 x int4, T >= 256,
# hidden and inter multiples of 256): 2 row tiles per projection, 8 K stages
# for gate/up, experts with more tokens than one 128-token tile.
SMALL_TC = TINY.with_(name="small_t300_int4_bf16", hidden=512, inter=256, afmt=A_BF16, T=300)

ALL = {w.name: w for w in [TINY, GLM_DECODE_T1, GLM_DECODE_T32_Q8, GLM_VERIFY_T4_BF16,
                           GLM_PREFILL_T2048_BF16, SMALL_TC, *sweep()]}
