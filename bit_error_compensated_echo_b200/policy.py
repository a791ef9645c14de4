"""Per-layer code width: which all-reduce calls run at 8 bits.

The pages' serving policy for Llama-3-8B promotes the earlier half of the
layers to 8-bit codes, which recovers most of the accuracy that 4 bits
loses there (ai4snews news summary, "Perspective").  The pages give the
fraction and the direction (the early layers) but no other rule, so the
policy here is that one: layer l of L runs at ``high`` bits when
l < round(promoted_fraction * L), else at ``low`` bits.  A layer holds
``sites_per_layer`` tensor-parallel all-reduce sites (two in a transformer
block: after attention and after the MLP), numbered in execution order.

Every width runs on one plan made with bits=8 and shares its compensator
state (``EchoPlan.allreduce(..., bits=policy.bits_for_site(s))``).
"""
from __future__ import annotations


class LayerPolicy:
    def __init__(self, n_layers: int, sites_per_layer: int = 2, promoted_fraction: float = 0.5,
                 high: int = 8, low: int = 4):
        if n_layers < 1 or sites_per_layer < 1 or not 0.0 <= promoted_fraction <= 1.0:
            raise ValueError("n_layers, sites_per_layer >= 1 and a fraction in [0, 1]")
        if high not in (4, 8) or low not in (4, 8):
            raise ValueError("code widths are 4 or 8")
        self.n_layers, self.sites_per_layer = int(n_layers), int(sites_per_layer)
        self.promoted = int(round(promoted_fraction * n_layers))
        self.high, self.low = int(high), int(low)

    @property
    def sites(self) -> int:
        return self.n_layers * self.sites_per_layer

    def bits_for_layer(self, layer: int) -> int:
        if not 0 <= layer < self.n_layers:
            raise IndexError("layer %d of %d" % (layer, self.n_layers))
        return self.high if layer < self.promoted else self.low

    def bits_for_site(self, site: int) -> int:
        """Width of the all-reduce at ``site`` (0-based, execution order;
        sites past the last layer wrap around, as the next step starts)."""
        return self.bits_for_layer((site % self.sites) // self.sites_per_layer)

    def schedule(self):
        return [self.bits_for_site(s) for s in range(self.sites)]
