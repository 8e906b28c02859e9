"""Workload shapes of one block-diffusion denoising step of the LLaDA2.0-Uni MoE dLLM backbone.

Each workload is named for what it is. The shapes follow the backbone as the LLaDA2.0-Uni paper review
(baba9811.github.io, section "MoE 백본과 Block-wise Attention") and the HF-mirror README (ai.gitcode.com,
sections on usage and "SPRINT 加速技术") describe its use: block length 32, 8 steps per block for text-to-image
with cfg 2.0, 32 steps per block with threshold acceptance for understanding, SPRINT prefix retention at 50 %.
The pages give no layer dimensions; the dimensions below are the stated workload sizes of this library.
"""
from dataclasses import dataclass, replace
import math


@dataclass(frozen=True)
class Workload:
    name: str
    dtype: str            # "bf16" or "f32": storage type of weights and activations
    n_layers: int
    H: int                # hidden size
    Hq: int               # query heads
    Hkv: int              # key/value heads
    d: int                # head dim
    E: int                # routed experts
    k: int                # experts per token
    I: int                # expert intermediate size (routed and shared)
    V: int                # vocabulary rows of the LM head
    B: int                # batch rows (each guidance row counts as a row)
    P: int                # cached prefix length before the block
    L: int                # block length
    T_s: int              # denoising steps per block
    mode: int = 0         # 0 = fixed schedule, 1 = threshold acceptance
    tau: float = 0.9
    k_max: int = 8
    cfg: int = 0          # 1: rows [0, B/2) conditional, [B/2, B) unconditional; 2 (editing): rows [0, B/3) on
                          # instruction and image, [B/3, 2B/3) on the image only, [2B/3, B) unconditional
    cfg_scale: float = 2.0   # two-way scale, or the text scale of editing guidance
    vocab_offset: int = 0 # first LM-head row scored (image-token slice)
    vocab_len: int = 0    # rows scored; 0 = all V
    sprint: int = 0       # SPRINT prefix retention at the first step of each block
    keep_ratio: float = 1.0
    rope_base: float = 10000.0
    eps: float = 1e-6
    w_std: float = 0.02
    lm_std: float = 0.02
    bias_range: float = 0.1
    seed: int = 0
    wfmt: str = "bf16"    # "fp8": expert and LM-head weights as E4M3 codes with per-row fp32 scales
    score: int = 0        # ranking of the masked positions: 0 largest probability, 1 top-2 margin, 2 negated entropy
    sprint_alpha: float = 1.0   # SPRINT importance = alpha * key norm + (1 - alpha) * confidence
    n_img_prefix: int = 0       # > 0: the first n_img_prefix prefix positions are image tokens (modality counts)
    img_keep_ratio: float = 1.0 # with image positions: keep ceil(ratio * n_img) of them, the rest of n_keep text
    cfg_image_scale: float = 1.0  # editing guidance (cfg 2): the image scale

    def __post_init__(self):
        # SPRINT serves no guidance and two-way guidance; under editing guidance it falls back to the plain decode on
        # the full caches (HF-mirror README, note under "SPRINT 加速技术")
        if self.cfg == 2 and self.sprint:
            object.__setattr__(self, "sprint", 0)

    @property
    def Tk(self) -> int:
        return self.B * self.L

    @property
    def vlen(self) -> int:
        return self.vocab_len if self.vocab_len else self.V

    @property
    def mask_id(self) -> int:
        return self.V - 1

    @property
    def n_keep(self) -> int:
        if not self.sprint:
            return self.P
        if self.n_img_prefix:   # modality keep ratios: images at img_keep_ratio, text at keep_ratio
            return self.n_keep_img + int(math.ceil(self.keep_ratio * (self.P - self.n_img_prefix)))
        return int(math.ceil(self.keep_ratio * self.P))

    @property
    def n_keep_img(self) -> int:
        return int(math.ceil(self.img_keep_ratio * self.n_img_prefix)) if self.n_img_prefix else 0

    @property
    def cap(self) -> int:
        """Cache rows per (row, kv head): prefix plus one block."""
        return self.P + self.L


# tiny fp32 single layer: hidden 256, 4 heads x 64 (no GQA), 8 experts top-2 + shared, inter 128, vocab 1024,
# prefix 64, block 16, 4 steps of 4 tokens, batch 1
TINY_F32 = Workload("tiny-f32-1layer", "f32", 1, 256, 4, 4, 64, 8, 2, 128, 1024, 1, 64, 16, 4)

# one MoE dLLM layer in bf16: hidden 2048, 16 q heads x 128, 4 kv heads, 256 experts top-8 + shared, inter 512,
# vocab 157184, prefix 1024, block 32 all masked, batch 1, 8 steps
ONE_LAYER = Workload("moe-dllm-1layer-p1024-b1", "bf16", 1, 2048, 16, 4, 128, 256, 8, 512, 157184, 1, 1024, 32, 8)

# text-to-image: 20 layers, cond + uncond rows, 256-token text prefix, 4096 image tokens in blocks of 32 at
# 8 steps per block, image-token head of 16384 rows. The prefix length is that of the block being decoded; the
# middle of the image (2048 image tokens already committed) is the representative block.
T2I = Workload("t2i-20layer-cfg2-b2", "bf16", 20, 2048, 16, 4, 128, 256, 8, 512, 157184, 2, 256 + 2048, 32, 8,
               cfg=1, cfg_scale=2.0, vocab_offset=157184 - 16384, vocab_len=16384)

# image editing: 20 layers, three guidance rows (instruction and image, image only, unconditional), a 512 x 512
# source image as 256 tokens plus a 64-token instruction in the prefix, the 256 output image tokens in blocks of 32
# at 8 steps per block with text scale 4.0 (the README's editing example) and image scale 1.0; the middle block
# (128 output tokens committed) is the representative one
EDIT = Workload("edit-20layer-cfg3-b3", "bf16", 20, 2048, 16, 4, 128, 256, 8, 512, 157184, 3, 64 + 256 + 128, 32, 8,
                cfg=2, cfg_scale=4.0, cfg_image_scale=1.0, vocab_offset=157184 - 16384, vocab_len=16384)

# thinking mode: 20 layers, batch 8, 4096-token prefix, SPRINT keeps 50 % of the prefix by key norm,
# 32 steps per block
THINKING = Workload("thinking-20layer-b8-p4096-sprint50", "bf16", 20, 2048, 16, 4, 128, 256, 8, 512, 157184, 8,
                    4096, 32, 32, sprint=1, keep_ratio=0.5)

# understanding: 20 layers, batch 16, prefix 2560 image + 128 question tokens, threshold 0.9 with at most
# 8 tokens accepted per step, 32 steps per block. The logit spread is widened so that confidences cross 0.9.
UNDERSTANDING = Workload("understanding-20layer-b16-p2688-thr0.9", "bf16", 20, 2048, 16, 4, 128, 256, 8, 512,
                         157184, 16, 2688, 32, 32, mode=1, tau=0.9, k_max=8, lm_std=0.2)

# compute-bound prefill of the thinking-mode prompt: 1 layer, 8 rows x 4096 tokens under the block-causal mask
PREFILL = Workload("prefill-1layer-b8-4096", "bf16", 1, 2048, 16, 4, 128, 256, 8, 512, 157184, 8, 0, 4096, 1)

# the same two workloads with the FP8 checkpoint's expert and LM-head weights (E4M3 codes, per-row scales)
ONE_LAYER_FP8 = replace(ONE_LAYER, name="moe-dllm-1layer-p1024-b1-fp8", wfmt="fp8")
UNDERSTANDING_FP8 = replace(UNDERSTANDING, name="understanding-20layer-b16-p2688-thr0.9-fp8", wfmt="fp8")

# one layer of the understanding workload (its batch, prefix and vocabulary): the size a profiler capture of the
# step's kernels takes (a few GB on the device)
UNDERSTANDING_1LAYER = replace(UNDERSTANDING, name="understanding-1layer-b16-p2688-thr0.9", n_layers=1)

ALL = [TINY_F32, ONE_LAYER, T2I, EDIT, THINKING, UNDERSTANDING, PREFILL, ONE_LAYER_FP8, UNDERSTANDING_FP8,
       UNDERSTANDING_1LAYER]
BY_NAME = {w.name: w for w in ALL}


def scaled(w: Workload, **kw) -> Workload:
    """Same workload with some sizes replaced (small parity cases)."""
    return replace(w, **kw)
