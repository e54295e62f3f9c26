"""Device-resident synthetic layers: one slab of (n_experts + 1) experts per
layer (shared expert last), filled on the GPU by the device generator, plus
the fp32 router weight and bias generated on the host and copied over.
Bytes equal those of synth.expert / synth.router for the same key."""
import numpy as np

import synth


def expert_offsets(shape):
    """Byte offset of each tensor inside one expert blob (16-byte aligned)."""
    offs, off = {}, 0
    for name, dt, shp, tag in synth.expert_layout(shape):
        offs[name] = off
        off += int(np.prod(shp)) * np.dtype(dt).itemsize
    assert off == shape.expert_bytes
    return offs


class DeviceLayer:
    """Synthetic layer `layer` of `seed` on the current CUDA device."""

    def __init__(self, shape, seed, layer, device="cuda", stream=None, routed=True):
        """routed=False: router, bias and shared expert only (the routed
        experts live elsewhere, e.g. in a pinned host store)."""
        import torch
        self.shape, self.seed, self.layer = shape, seed, layer
        n = shape.n_experts + shape.n_shared
        ids = list(range(n)) if routed else list(range(shape.n_experts, n))
        self.slab = torch.empty(max(1, len(ids)) * shape.expert_bytes, dtype=torch.uint8,
                                device=device)
        base = self.slab.data_ptr()
        offs = expert_offsets(shape)
        st = (stream or torch.cuda.current_stream()).cuda_stream
        self.experts = [None] * n
        for i, e in enumerate(ids):
            ptrs = {k: base + i * shape.expert_bytes + o for k, o in offs.items()}
            synth.fill_expert_device(shape, seed, layer, e, ptrs, st)
            self.experts[e] = ptrs
        w, b = synth.router(shape, seed, layer)
        self.w_router = torch.from_numpy(w).to(device)
        self.bias = torch.from_numpy(b).to(device)

    @property
    def routed(self):
        return self.experts[: self.shape.n_experts]

    @property
    def shared(self):
        return self.experts[self.shape.n_experts] if self.shape.n_shared else None

    def host_expert(self, e):
        """Host copy of expert e (regenerated on the host, not read back)."""
        return synth.expert(self.shape, self.seed, self.layer, e)

    def host_router(self):
        return synth.router(self.shape, self.seed, self.layer)
