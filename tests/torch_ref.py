"""The encoder written with PyTorch library routines (CPU, fp64).

Used only to pin the C oracle: its convolutions are ``torch.nn.functional.
conv2d``, its norms ``layer_norm``, its attention ``scaled_dot_product_
attention`` with a boolean window mask, its activations ``gelu`` / ``silu``.
A mistake in the oracle's own loops (a transposed kernel, a dropped bias, a
wrong index) shows up as a disagreement with these routines.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

from audio_encoder_b200 import synth


class TorchRef:
    def __init__(self, blob: np.ndarray, n_layers: int):
        table, _ = synth.weight_offsets(n_layers)
        f32 = synth.bf16_bits_to_f32(blob)
        self.n_layers = n_layers
        self.w = {}
        for name, (off, shape) in table.items():
            n = int(np.prod(shape))
            self.w[name] = torch.from_numpy(f32[off:off + n].astype(np.float64).reshape(shape))

    def positions(self, T: int) -> torch.Tensor:
        half = 640
        inv = torch.exp(-torch.arange(half, dtype=torch.float64) * (np.log(10000.0) / (half - 1)))
        t = torch.arange(T, dtype=torch.float64)[:, None] * inv[None, :]
        return torch.cat([torch.sin(t), torch.cos(t)], dim=1)

    def stem_chunk(self, mel_norm: np.ndarray) -> torch.Tensor:
        W = self.w
        fc = mel_norm.shape[0]
        img = torch.zeros(1, 1, 128, 800, dtype=torch.float64)
        img[0, 0, :, :fc] = torch.from_numpy(mel_norm.astype(np.float64)).T
        x = F.gelu(F.conv2d(img, W["conv1.weight"], W["conv1.bias"], stride=2, padding=1))
        x = F.gelu(F.conv2d(x, W["conv2.weight"], W["conv2.bias"], stride=2, padding=1))
        x = F.gelu(F.conv2d(x, W["conv3.weight"], W["conv3.bias"], stride=2, padding=1))
        # [1, 480, 16, 100] -> [100, 480*16] with index c*16 + f
        x = x[0].permute(2, 0, 1).reshape(100, 480 * 16)
        tc = -(-fc // 8)
        y = F.linear(x[:tc], W["conv_out.weight"])
        return y + self.positions(tc)

    @staticmethod
    def e4m3_rows(x64: torch.Tensor):
        """Per-row e4m3 operands of x (fp32 values): scale = row max / 448 in
        fp32, values rounded by torch's float8_e4m3fn conversion."""
        x = x64.to(torch.float32)
        s = x.abs().amax(dim=1) / 448.0
        safe = torch.where(s > 0, s, torch.ones_like(s))
        q = (x / safe[:, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn).to(torch.float64)
        q = torch.where(s[:, None] > 0, q, torch.zeros_like(q))
        return q, s.to(torch.float64)

    def linear_e4m3(self, h: torch.Tensor, w: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
        a8, sa = self.e4m3_rows(h)
        w8, sw = self.e4m3_rows(w)
        return (a8 @ w8.T) * sa[:, None] * sw[None, :] + b

    # E2M1 values with the even codes first, so that argmin settles a tie on
    # the even neighbour
    E2M1_EVEN_FIRST = torch.tensor([0.0, 1.0, 2.0, 4.0, 0.5, 1.5, 3.0, 6.0], dtype=torch.float32)

    @classmethod
    def nvfp4_rows(cls, x64: torch.Tensor, per_row: bool):
        """NVFP4 operands of x (fp32 values): g = amax / 2688 per row or per
        tensor, block scales of 16 by torch's float8_e4m3fn conversion, E2M1
        values by nearest-on-the-grid (ties to the even code, +-6 saturates).
        Returns (q * s_b as fp64, g as fp64 [rows] or scalar)."""
        x = x64.to(torch.float32)
        rows, cols = x.shape
        amax = x.abs().amax(dim=1) if per_row else x.abs().amax().expand(rows)
        g = amax / 2688.0
        xb = x.view(rows, cols // 16, 16)
        bmax = xb.abs().amax(dim=2)
        safe_g = torch.where(g > 0, g, torch.ones_like(g))
        sb = (bmax / (safe_g[:, None] * 6.0)).clamp(max=448.0).to(torch.float8_e4m3fn).to(torch.float32)
        sb = torch.where(g[:, None] > 0, sb, torch.zeros_like(sb))
        sg = sb * g[:, None]
        y = xb / torch.where(sg > 0, sg, torch.ones_like(sg))[:, :, None]
        d = (y.abs()[..., None] - cls.E2M1_EVEN_FIRST).abs()
        q = cls.E2M1_EVEN_FIRST[d.argmin(dim=-1)] * torch.sign(y)
        q = torch.where(sg[:, :, None] > 0, q, torch.zeros_like(q))
        unit = (q * sb[:, :, None]).view(rows, cols)
        return unit.to(torch.float64), g.to(torch.float64)

    def linear_nvfp4(self, h: torch.Tensor, w: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
        ua, ga = self.nvfp4_rows(h, per_row=True)
        uw, gw = self.nvfp4_rows(w, per_row=False)
        return (ua @ uw.T) * ga[:, None] * gw[0] + b

    def layers(self, x: torch.Tensor, windows, l0=0, l1=None, fp8=False, nvfp4=False) -> torch.Tensor:
        W = self.w
        lin = (self.linear_nvfp4 if nvfp4 else self.linear_e4m3 if fp8
               else (lambda h, w, b: F.linear(h, w, b)))
        T = x.shape[0]
        wid = torch.empty(T, dtype=torch.long)
        for i in range(len(windows) - 1):
            wid[windows[i]:windows[i + 1]] = i
        mask = wid[:, None] == wid[None, :]
        l1 = self.n_layers if l1 is None else l1
        for l in range(l0, l1):
            p = f"layers.{l}."
            h = F.layer_norm(x, (1280,), W[p + "ln1.weight"], W[p + "ln1.bias"], eps=1e-5)
            q = lin(h, W[p + "q.weight"], W[p + "q.bias"]).view(T, 20, 64).transpose(0, 1)
            k = lin(h, W[p + "k.weight"], W[p + "k.bias"]).view(T, 20, 64).transpose(0, 1)
            v = lin(h, W[p + "v.weight"], W[p + "v.bias"]).view(T, 20, 64).transpose(0, 1)
            a = F.scaled_dot_product_attention(q, k, v, attn_mask=mask)
            a = a.transpose(0, 1).reshape(T, 1280)
            x = x + F.linear(a, W[p + "o.weight"], W[p + "o.bias"])
            h = F.layer_norm(x, (1280,), W[p + "ln2.weight"], W[p + "ln2.bias"], eps=1e-5)
            f = F.gelu(lin(h, W[p + "fc1.weight"], W[p + "fc1.bias"]))
            x = x + F.linear(f, W[p + "fc2.weight"], W[p + "fc2.bias"])
        return x

    def head(self, x: torch.Tensor) -> torch.Tensor:
        W = self.w
        h = F.layer_norm(x, (1280,), W["ln_post.weight"], W["ln_post.bias"], eps=1e-5)
        h = F.gelu(F.linear(h, W["proj1.weight"], W["proj1.bias"]))
        return F.linear(h, W["proj2.weight"], W["proj2.bias"])

    def adapter(self, h: torch.Tensor) -> torch.Tensor:
        W = self.w
        g = F.linear(h, W["adapter.gate.weight"], W["adapter.gate.bias"])
        u = F.linear(h, W["adapter.up.weight"], W["adapter.up.bias"])
        return F.linear(F.silu(g) * u, W["adapter.down.weight"], W["adapter.down.bias"])
