"""Synthetic MoE layers resident in device memory.

Draws codes and scales with the device twin of the generator (bit-identical to
the host generator the oracle side uses) and packs them with the library's
device packer into one buffer per matrix kind, experts at a fixed stride.
Recipe (the workload shapes): routed gate/up ROCmFP2, routed down ROCmFP3,
shared expert ROCmFP4; codes uniform over the levels; scales 0.02*2^U(-1,1).
"""
from __future__ import annotations

import torch

import synth

ROUTED_KINDS = (synth.KIND_GATE, synth.KIND_UP, synth.KIND_DOWN)
SHARED_KINDS = (synth.KIND_SH_GATE, synth.KIND_SH_UP, synth.KIND_SH_DOWN)


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class SynthLayer:
    """Packed device buffers of one synthetic layer (seed, layer)."""

    def __init__(self, seed: int, layer: int, H: int, I: int, E: int, k: int, fmts=(2, 2, 3), shared_fmts=(4, 4, 4),
                 has_shared: bool = True, device="cuda", experts=None, mix=None):
        """mix: ROCmFPX MIX, E pairs (gate/up format, down format), one per
        routed expert; the experts are then packed back to back (256-byte
        aligned) and `fmts` is ignored."""
        import block_quantized_moe_rocmfpx_b200 as rfx
        self.seed, self.layer, self.H, self.I, self.E, self.k = seed, layer, H, I, E, k
        self.fmts, self.shared_fmts, self.has_shared = tuple(fmts), tuple(shared_fmts), has_shared
        self.mix = None if mix is None else [(int(a), int(a), int(b)) for a, b in mix]
        shapes = ((I, H), (I, H), (H, I))
        if self.mix is None:
            self.expert_fmts = [self.fmts] * E
            self.strides = tuple(_align(rfx.rfx_packed_bytes(f, r, c)) for f, (r, c) in zip(fmts, shapes))
            self.offsets = [[e * s for e in range(E)] for s in self.strides]
            sizes = [E * s for s in self.strides]
        else:
            assert len(self.mix) == E
            self.expert_fmts = self.mix
            self.strides = (0, 0, 0)
            self.offsets, sizes = [], []
            for i, (r, c) in enumerate(shapes):
                off, o = [], 0
                for e in range(E):
                    off.append(o)
                    o += _align(rfx.rfx_packed_bytes(self.mix[e][i], r, c))
                self.offsets.append(off)
                sizes.append(o)
        self.bufs = [torch.empty(n, dtype=torch.uint8, device=device) for n in sizes]
        cmax = max(H, I) * max(H, I)
        codes = torch.empty(cmax, dtype=torch.uint8, device=device)
        scales = torch.empty(cmax // 32 * 2, dtype=torch.uint8, device=device)
        todo = range(E) if experts is None else experts
        for e in todo:
            for i, (kind, (r, c), buf) in enumerate(zip(ROUTED_KINDS, shapes, self.bufs)):
                f = self.expert_fmts[e][i]
                o = self.offsets[i][e]
                self._gen(kind, e, f, r, c, codes, scales, buf[o:o + _align(rfx.rfx_packed_bytes(f, r, c))])
        self.shared = None
        if has_shared:
            self.shared = []
            for kind, f, (r, c) in zip(SHARED_KINDS, shared_fmts, shapes):
                buf = torch.empty(_align(rfx.rfx_packed_bytes(f, r, c)), dtype=torch.uint8, device=device)
                self._gen(kind, 0, f, r, c, codes, scales, buf)
                self.shared.append(buf)
        torch.cuda.synchronize()
        self.expert_bytes = [sum(rfx.rfx_packed_bytes(f, r, c) for f, (r, c) in zip(self.expert_fmts[e], shapes))
                             for e in range(E)]
        self.packed_bytes_per_expert = self.expert_bytes[0]
        self.shared_bytes = sum(rfx.rfx_packed_bytes(f, r, c) for f, (r, c) in zip(shared_fmts, shapes)) \
            if has_shared else 0

    def _gen(self, kind, e, f, rows, cols, codes, scales, dst):
        import block_quantized_moe_rocmfpx_b200 as rfx
        spec = synth.MatrixSpec(self.seed, self.layer, kind, e, f, rows, cols)
        synth.codes_dev(spec.code_key, f, rows, cols, codes)
        synth.scales_dev(spec.scale_key, f, rows, cols, scales)
        rfx.rfx_pack_device(f, codes, scales, rows, cols, dst)

    def spec(self, kind: int, expert: int) -> synth.MatrixSpec:
        H, I = self.H, self.I
        routed = kind in ROUTED_KINDS
        idx = (ROUTED_KINDS if routed else SHARED_KINDS).index(kind)
        f = (self.expert_fmts[expert] if routed else self.shared_fmts)[idx]
        r, c = ((I, H), (I, H), (H, I))[idx]
        return synth.MatrixSpec(self.seed, self.layer, kind, expert if routed else 0, f, r, c)

    def moe_layer(self, max_T: int = 8, bufs=None, shared=None):
        """The library's layer handle over these buffers (or over copies of
        them with the same layout: bufs, shared)."""
        import block_quantized_moe_rocmfpx_b200 as rfx
        bufs = self.bufs if bufs is None else bufs
        shared = self.shared if shared is None else shared
        mix = None
        if self.mix is not None:
            mix = [(self.mix[e][0], self.mix[e][2], self.offsets[0][e], self.offsets[1][e], self.offsets[2][e])
                   for e in range(self.E)]
        return rfx.MoeLayer(self.H, self.I, self.E, self.k, self.fmts, *bufs, self.strides,
                            shared=shared, shared_fmts=self.shared_fmts, max_T=max_T, mix=mix)

    def union_bytes(self, experts) -> int:
        """Packed weight bytes one pass reads for the given union of routed experts."""
        return sum(self.expert_bytes[e] for e in set(int(e) for e in experts)) + self.shared_bytes


def heat_mix(seed: int, layer: int, E: int, zipf_s: float):
    """ROCmFPX MIX chosen by routing heat: experts ranked by their Zipf
    popularity; the hottest eighth FP4 gate/up and FP4 down, the next three
    eighths FP3 / FP3, the rest FP2 / FP3 (the uniform layer's assignment)."""
    import numpy as np
    order = np.argsort(-synth.zipf_bias(seed, layer, E, zipf_s), kind="stable")
    mix = [(2, 3)] * E
    for r, e in enumerate(order):
        if r < E // 8:
            mix[e] = (4, 4)
        elif r < E // 2:
            mix[e] = (3, 3)
    return mix
