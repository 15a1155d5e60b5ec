"""Layer-wise Mix'n'Match: which width each layer of a stack is served at.

One packed model serves every width, so a stack can give each layer its own r
("Matryoshka Quantization | Summary", §4.3 Layerwise Mix'n'Match; MatGPTQ §5.4).  The pages
compare four allocation strategies -- Pyramid (higher precision in the middle layers, lower
near the first and last), Reverse Pyramid, Increasing and Decreasing (precision rising or
falling with depth) -- and report Pyramid as the best of them (same Summary page, App. B), and
they measure a configuration by its effective bits per FFN parameter, the average precision
assigned to those weights (§4.3).  They print no allocation procedure.  The reading here:
  * a strategy is an order of the layers, the ones that get more precision first (ties in the
    order go to the shallower layer);
  * for a budget of effective bits, every layer starts at the narrowest width and the layers,
    in that order, each take the widest width that keeps the parameter-weighted mean within the
    budget.  The result is maximal: raising any one layer to a wider width would break it.
Host logic only (a list of widths); the kernels take r per call.
"""

from __future__ import annotations

WIDTHS = (2, 3, 4, 6, 8)
STRATEGIES = ("pyramid", "reverse_pyramid", "increasing", "decreasing")
METADATA_BITS_PER_GROUP = 24  # one fp16 scale and one uint8 zero point per group


def layer_order(n_layers: int, strategy: str = "pyramid") -> list:
    """Layer indices in the order they receive precision under `strategy`."""
    if n_layers < 1:
        raise ValueError("n_layers must be >= 1")
    mid = (n_layers - 1) / 2.0
    keys = {
        "pyramid": lambda l: (abs(l - mid), l),
        "reverse_pyramid": lambda l: (-abs(l - mid), l),
        "increasing": lambda l: (-l,),
        "decreasing": lambda l: (l,),
    }
    if strategy not in keys:
        raise ValueError(f"unknown strategy {strategy!r}; one of {STRATEGIES}")
    return sorted(range(n_layers), key=keys[strategy])


def allocate_widths(n_layers: int, target_bits: float, strategy: str = "pyramid", widths=(2, 4, 8),
                    sizes=None) -> list:
    """Per-layer widths whose parameter-weighted mean is at most `target_bits`.

    widths: the widths a layer may take (each in {2, 3, 4, 6, 8}); sizes: parameters per layer
    (default: equal).  Greedy in `layer_order(n_layers, strategy)`: each layer takes the widest
    width that fits the budget left with the remaining layers at the narrowest width."""
    ws = sorted(set(int(r) for r in widths))
    if not ws or any(r not in WIDTHS for r in ws):
        raise ValueError("widths must be a non-empty subset of (2, 3, 4, 6, 8)")
    sizes = [1] * n_layers if sizes is None else [int(v) for v in sizes]
    if len(sizes) != n_layers or any(v <= 0 for v in sizes):
        raise ValueError("one positive size per layer")
    total = sum(sizes)
    if not ws[0] <= target_bits:
        raise ValueError(f"target_bits {target_bits} is below the narrowest width {ws[0]}")
    # integer bookkeeping: bits granted above the narrowest width
    budget = int(target_bits * total + 1e-9) - ws[0] * total
    out = [ws[0]] * n_layers
    for l in layer_order(n_layers, strategy):
        for r in reversed(ws[1:]):
            extra = (r - ws[0]) * sizes[l]
            if extra <= budget:
                out[l] = r
                budget -= extra
                break
    return out


def effective_bits(layer_widths, sizes=None, group: int | None = None) -> float:
    """Average bits per weight of a stack served at `layer_widths`, weighted by the parameters
    of each layer (sizes, default equal).  With `group`, the scale and zero point each group of
    `group` weights carries (16 + 8 bits) are counted too: r + 24/group bits a weight."""
    rs = [float(r) for r in layer_widths]
    sizes = [1.0] * len(rs) if sizes is None else [float(v) for v in sizes]
    if not rs or len(sizes) != len(rs):
        raise ValueError("one size per layer")
    meta = METADATA_BITS_PER_GROUP / float(group) if group else 0.0
    return sum((r + meta) * n for r, n in zip(rs, sizes)) / sum(sizes)
