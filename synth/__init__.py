"""Seeded synthetic inputs shared by the CPU oracle and the CUDA library.

This module only draws random numbers and names model shapes; it holds none
of the decode step's arithmetic.  Every tensor is a pure function of
(seed, tensor id, shape, device kind): weights N(0, 0.02^2), norm gains
1 + N(0, 0.01^2), KV prefill N(0, 1), embeddings N(0, 0.02^2), as the
workload descriptions fix them.  Values are drawn by torch's generators
(CPU or CUDA) in fp32 and rounded to bf16, so a tensor drawn on the GPU
is not the same as one drawn on the CPU with the same seed: a test draws
each input once and hands the same bytes to both sides.
"""
from __future__ import annotations

import dataclasses
import hashlib

import torch


@dataclasses.dataclass(frozen=True)
class BodyShape:
    """Shape of the Qwen3-style Global LLM and its sampleable vocab slice."""
    hidden: int
    n_layers: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    slice_start: int
    slice_len: int
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6
    end_token: int = -1  # vocab row of the end token, sampleable with the slice; -1: none


@dataclasses.dataclass(frozen=True)
class DepthShape:
    """Shape of the RVQ depth decoder (MHA: as many KV heads as query heads)."""
    hidden: int = 1024
    n_layers: int = 4
    n_heads: int = 16
    head_dim: int = 64
    ffn: int = 2816
    codebooks: int = 7
    vocab: int = 1024
    sem_vocab: int = 16384
    in_hidden: int = 4096
    rope_theta: float = 1.0e6
    rms_eps: float = 1.0e-6


# Tiny 1-layer decode checked over 16 consecutive frames.
TINY = BodyShape(hidden=256, n_layers=1, n_q_heads=4, n_kv_heads=2, head_dim=64, ffn=768,
                 vocab=2048, slice_start=1024, slice_len=512)
# One Qwen3-8B decoder layer (GEMV roofline microbench); no lm_head of its own.
LAYER8B = BodyShape(hidden=4096, n_layers=1, n_q_heads=32, n_kv_heads=8, head_dim=128,
                    ffn=12288, vocab=200000, slice_start=151675, slice_len=16384)
# The full 36-layer 8B body with its sliced lm_head.
FULL8B = BodyShape(hidden=4096, n_layers=36, n_q_heads=32, n_kv_heads=8, head_dim=128,
                   ffn=12288, vocab=200000, slice_start=151675, slice_len=16384)
# The same with the end token sampleable (the generation loop's stop code).
FULL8B_END = dataclasses.replace(FULL8B, end_token=151670)
# TINY with an end token four rows below the code block, as in the 8B vocab.
TINY_END = dataclasses.replace(TINY, end_token=1019)
DEPTH = DepthShape()

LAYER_TENSORS = ("attn_norm", "wq", "wk", "wv", "q_norm", "k_norm", "wo", "mlp_norm",
                 "wg", "wu", "wd")
NORM_TENSORS = ("attn_norm", "q_norm", "k_norm", "mlp_norm")


def _stream_seed(seed: int, name: str) -> int:
    h = hashlib.sha256(f"{int(seed)}/{name}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, name: str, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev.type if dev.type != "cuda" else dev)
    g.manual_seed(_stream_seed(seed, name))
    return g


def normal(shape, seed: int, name: str, std: float = 1.0, mean: float = 0.0,
           device="cpu", dtype=torch.bfloat16) -> torch.Tensor:
    """N(mean, std^2) drawn in fp32 from the stream (seed, name), cast to dtype."""
    g = _gen(seed, name, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(dtype)


def layer_shapes(s) -> dict:
    H, d = s.hidden, s.head_dim
    hq = s.n_q_heads if isinstance(s, BodyShape) else s.n_heads
    hkv = s.n_kv_heads if isinstance(s, BodyShape) else s.n_heads
    return {
        "attn_norm": (H,), "wq": (hq * d, H), "wk": (hkv * d, H), "wv": (hkv * d, H),
        "q_norm": (d,), "k_norm": (d,), "wo": (H, hq * d), "mlp_norm": (H,),
        "wg": (s.ffn, H), "wu": (s.ffn, H), "wd": (H, s.ffn),
    }


def layer_weights(s, seed: int, layer: int, device="cpu", prefix: str = "body") -> dict:
    """One decoder layer's bf16 tensors (weights N(0,.02^2), gains 1+N(0,.01^2))."""
    out = {}
    for name, shape in layer_shapes(s).items():
        tag = f"{prefix}/L{layer}/{name}"
        if name in NORM_TENSORS:
            out[name] = normal(shape, seed, tag, std=0.01, mean=1.0, device=device)
        else:
            out[name] = normal(shape, seed, tag, std=0.02, device=device)
    return out


def final_norm(s, seed: int, device="cpu", prefix: str = "body") -> torch.Tensor:
    return normal((s.hidden,), seed, f"{prefix}/final_norm", std=0.01, mean=1.0, device=device)


def lm_head_rows(s: BodyShape, seed: int, row0: int, nrows: int, device="cpu") -> torch.Tensor:
    """Rows [row0, row0+nrows) of the full [vocab, hidden] lm_head, drawn in
    blocks of 1024 vocab rows so that any slice equals the same rows of the
    full matrix."""
    blocks = []
    b0, b1 = row0 // 1024, (row0 + nrows - 1) // 1024
    for b in range(b0, b1 + 1):
        n = min(1024, s.vocab - b * 1024)
        blocks.append(normal((n, s.hidden), seed, f"lm_head/block{b}", std=0.02, device=device))
    full = torch.cat(blocks, 0)
    off = row0 - b0 * 1024
    return full[off:off + nrows].contiguous()


def lm_head_slice(s: BodyShape, seed: int, device="cpu") -> torch.Tensor:
    return lm_head_rows(s, seed, s.slice_start, s.slice_len, device)


def lm_head_full(s: BodyShape, seed: int, device="cpu") -> torch.Tensor:
    return lm_head_rows(s, seed, 0, s.vocab, device)


def lm_head_end_row(s: BodyShape, seed: int, device="cpu") -> torch.Tensor:
    """The end token's row [hidden] of the full lm_head."""
    return lm_head_rows(s, seed, s.end_token, 1, device)[0].contiguous()


def embedding(s: BodyShape, seed: int, device="cpu") -> torch.Tensor:
    """Token-embedding table [vocab, hidden] used to feed a drawn code back."""
    return normal((s.vocab, s.hidden), seed, "embed_tokens", std=0.02, device=device)


def embedding_slice(s: BodyShape, seed: int, device="cpu") -> torch.Tensor:
    """The code block's rows [slice_len, hidden] of a token-embedding table,
    drawn in blocks of 1024 vocab rows (the generation loop's feedback table;
    not the same values as embedding())."""
    blocks = []
    b0, b1 = s.slice_start // 1024, (s.slice_start + s.slice_len - 1) // 1024
    for b in range(b0, b1 + 1):
        n = min(1024, s.vocab - b * 1024)
        blocks.append(normal((n, s.hidden), seed, f"embed_tokens/block{b}", std=0.02,
                             device=device))
    off = s.slice_start - b0 * 1024
    return torch.cat(blocks, 0)[off:off + s.slice_len].contiguous()


def audio_embeddings(d: DepthShape, hidden: int, seed: int, device="cpu") -> list:
    """The residual codebooks' audio-embedding tables, d.codebooks x [d.vocab, hidden]."""
    return [normal((d.vocab, hidden), seed, f"audio_emb{j}", std=0.02, device=device)
            for j in range(d.codebooks)]


def kv_prefill(s, rows: int, n_pos: int, seed: int, device="cpu"):
    """Per-row prefilled cache contents N(0,1), layout [rows, layers, n_pos, Hkv, d]
    for K and for V (the prefill stands for already-rotated keys)."""
    hkv = s.n_kv_heads if isinstance(s, BodyShape) else s.n_heads
    ks, vs = [], []
    for r in range(rows):
        ks.append(normal((s.n_layers, n_pos, hkv, s.head_dim), seed + 1000 + r, "kv/K",
                         device=device))
        vs.append(normal((s.n_layers, n_pos, hkv, s.head_dim), seed + 1000 + r, "kv/V",
                         device=device))
    return torch.stack(ks, 0), torch.stack(vs, 0)


def frame_input(s, rows: int, seed: int, frame: int, device="cpu") -> torch.Tensor:
    """A frame's input embedding per row, N(0, 0.02^2) like the embedding tables."""
    return normal((rows, s.hidden), seed, f"x_in/frame{frame}", std=0.02, device=device)


def depth_weights(d: DepthShape, seed: int, device="cpu") -> dict:
    """Depth decoder bf16 tensors: layers, proj, embedding tables, final norm, heads."""
    out = {"layers": [layer_weights(d, seed, l, device, prefix="depth") for l in range(d.n_layers)]}
    out["proj"] = normal((d.hidden, d.in_hidden), seed, "depth/proj", std=0.02, device=device)
    out["emb"] = [normal((d.sem_vocab if j == 0 else d.vocab, d.hidden), seed, f"depth/emb{j}",
                         std=0.02, device=device) for j in range(d.codebooks)]
    out["final_norm"] = final_norm(d, seed, device, prefix="depth")
    out["heads"] = [normal((d.vocab, d.hidden), seed, f"depth/head{j}", std=0.02, device=device)
                    for j in range(d.codebooks)]
    return out


# ------------------------------------------------------------------- DiT ----

@dataclasses.dataclass(frozen=True)
class DitShape:
    """Shape of the chunk-denoise DiT (DiffSynth-Studio article, "各子模型的结构要点")."""
    width: int = 2048        # 32 heads x 64
    n_layers: int = 36
    n_heads: int = 32
    head_dim: int = 64
    ffn: int = 8192
    latent: int = 128        # Flow-VAE latent channels
    cond: int = 2048         # condition channels
    temb: int = 256          # Fourier timestep features
    rope_dims: int = 32      # rotated dims per head (partial rotary embedding)
    rope_theta: float = 1.0e4
    ln_eps: float = 1.0e-5


DIT = DitShape()
# A 200-frame chunk at the latent rate 44100 / 512 Hz: int(200 * 44100 / 512 / 25)
DIT_CHUNK_T = 689
DIT_TINY = DitShape(width=256, n_layers=2, n_heads=4, head_dim=64, ffn=512, latent=32, cond=192,
                    temb=32, rope_dims=32)

DIT_LAYER_TENSORS = ("ln1_g", "ln1_b", "wqkv", "wo", "ln2_g", "ln2_b", "wg", "wu", "wd")


def dit_layer_weights(s: DitShape, seed: int, layer: int, device="cpu") -> dict:
    """One DiT block's fp16 tensors: weights N(0, .02^2), LayerNorm gains
    1 + N(0, .01^2) and biases N(0, .01^2)."""
    W, F = s.width, s.ffn
    shapes = {"ln1_g": (W,), "ln1_b": (W,), "wqkv": (3 * W, W), "wo": (W, W), "ln2_g": (W,),
              "ln2_b": (W,), "wg": (F, W), "wu": (F, W), "wd": (W, F)}
    out = {}
    for name, shape in shapes.items():
        tag = f"dit/L{layer}/{name}"
        if name.endswith("_g"):
            out[name] = normal(shape, seed, tag, std=0.01, mean=1.0, device=device,
                               dtype=torch.float16)
        elif name.endswith("_b"):
            out[name] = normal(shape, seed, tag, std=0.01, device=device, dtype=torch.float16)
        else:
            out[name] = normal(shape, seed, tag, std=0.02, device=device, dtype=torch.float16)
    return out


def dit_weights(s: DitShape, seed: int, device="cpu", layers=None) -> dict:
    """The DiT's fp16 tensors outside the blocks, plus the blocks (all of them,
    or the given list)."""
    W, Cin = s.width, 2 * s.latent + s.cond
    f16 = torch.float16
    return {
        "w_in": normal((W, Cin), seed, "dit/w_in", std=0.02, device=device, dtype=f16),
        "w_t1": normal((W, s.temb), seed, "dit/w_t1", std=0.02, device=device, dtype=f16),
        "w_t2": normal((W, W), seed, "dit/w_t2", std=0.02, device=device, dtype=f16),
        "layers": layers if layers is not None else
        [dit_layer_weights(s, seed, l, device) for l in range(s.n_layers)],
        "lnf_g": normal((W,), seed, "dit/lnf_g", std=0.01, mean=1.0, device=device, dtype=f16),
        "lnf_b": normal((W,), seed, "dit/lnf_b", std=0.01, device=device, dtype=f16),
        "w_out": normal((s.latent, W), seed, "dit/w_out", std=0.02, device=device, dtype=f16),
    }


def dit_inputs(s: DitShape, T: int, seed: int, device="cpu"):
    """A chunk's step inputs: x_t [T, latent] fp32 N(0, 1) (the noisy latent),
    the context latent [T, latent] fp16 N(0, 1) over the first overlap frames
    (172 of a full chunk, proportionally fewer for short T) and zeros after,
    and the condition [T, cond] fp16 N(0, 1)."""
    x = normal((T, s.latent), seed, "dit/x_t", device=device, dtype=torch.float32)
    ctx = normal((T, s.latent), seed, "dit/ctx", device=device, dtype=torch.float16)
    n_ov = min(T, max(1, (172 * T) // DIT_CHUNK_T))
    ctx[n_ov:] = 0
    cond = normal((T, s.cond), seed, "dit/cond", device=device, dtype=torch.float16)
    return x, ctx, cond
