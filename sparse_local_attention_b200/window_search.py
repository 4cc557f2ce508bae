"""Per-head window search: for each attention head, the cheapest STA window
whose output stays within an error budget of a reference output.

"Fast Video Generation with Sliding Tile Attention", summary page
(Methodology, Technical Contribution, Limitations): the window size of each
head is configured automatically by profiling the attention's local patterns.
The pages give no procedure.  This module implements the plainest reading of
that step, on the caller's data: candidate windows are tried from the fewest
key tiles upwards, each with one sta_forward call over all heads, and every
head keeps the first candidate whose output O satisfies

    ||O_sta - O_ref||_F / ||O_ref||_F <= budget      (over batch, tokens, d)

against a reference O_ref that the caller supplies (or dense attention when
none is given).  A head that no candidate satisfies gets the whole tile grid,
where STA is full attention.  Profiling a pretrained video model is not part of
this: it needs the model's weights and prompts.

Attention itself runs in the library's kernels (sta_forward); the reference
and the error norms are plain torch operations on the caller's device.
"""
from dataclasses import dataclass, field
from typing import Callable, List, Optional, Sequence, Tuple

import torch

from . import sta

Window = Tuple[int, int, int]


@dataclass
class WindowSearchResult:
    windows: List[Window]            # chosen window per head
    errors: List[float]              # relative error of the chosen window per head
    keys_per_query: List[int]        # keys each query of the head attends to
    tried: List[Tuple[Window, List[float]]] = field(default_factory=list)  # (candidate, error per head)


def clamped_keys(window: Sequence[int], tile: Sequence[int], grid: Sequence[int]) -> int:
    """Keys per query for a window of tiles, each extent clamped to the grid."""
    n = 1
    for w, t, g in zip(window, tile, grid):
        n *= min(int(w), int(g)) * int(t)
    return n


def relative_errors(o: torch.Tensor, ref: torch.Tensor) -> List[float]:
    """||o - ref|| / ||ref|| per head for [batch, heads, tokens, d] tensors."""
    o64, r64 = o.double(), ref.double()
    num = (o64 - r64).pow(2).sum(dim=(0, 2, 3)).sqrt()
    den = r64.pow(2).sum(dim=(0, 2, 3)).sqrt().clamp_min(1e-300)
    return (num / den).tolist()


def dense_reference(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: float = 0.0) -> torch.Tensor:
    """Full (unmasked) attention over every token, the reference when the
    caller supplies none."""
    return torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=scale if scale > 0 else None)


def search_windows(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, T: int, H: int, W: int,
                   tile: Sequence[int], candidates: Sequence[Sequence[int]], budget: float,
                   reference: Optional[torch.Tensor] = None, scale: float = 0.0,
                   forward: Optional[Callable[[Window], torch.Tensor]] = None) -> WindowSearchResult:
    """Choose a window per head.

    q, k, v: [batch, heads, T*H*W, d] bf16 in raster token order.  candidates:
    windows in tiles (w_t, w_h, w_w), tried in order of clamped key count
    (ties in the given order).  reference: the output to stay close to (same
    shape as q); dense attention when None.  forward(window) -> O replaces the
    library call (used to test the selection on its own)."""
    if budget < 0:
        raise ValueError("budget must be >= 0")
    if not candidates:
        raise ValueError("no candidate windows")
    B, heads, N, d = q.shape
    if N != T * H * W:
        raise ValueError(f"token count {N} != T*H*W = {T * H * W}")
    grid = (T // tile[0], H // tile[1], W // tile[2])
    full: Window = tuple(grid)  # type: ignore[assignment]
    order = sorted(range(len(candidates)), key=lambda i: (clamped_keys(candidates[i], tile, grid), i))

    if forward is None:
        def forward(window: Window) -> torch.Tensor:
            problem = sta.Problem(B, heads, d, T, H, W, tuple(tile), [tuple(window)] * heads, scale)
            plan = sta.sta_plan_create(problem)
            try:
                o, _ = sta.sta_forward(plan, q, k, v, check=True, want_lse=False)
            finally:
                plan.destroy()
            return o

    if reference is None:
        reference = dense_reference(q, k, v, scale)

    chosen: List[Optional[Window]] = [None] * heads
    chosen_err: List[float] = [float("nan")] * heads
    tried: List[Tuple[Window, List[float]]] = []
    for i in order:
        window: Window = tuple(int(x) for x in candidates[i])  # type: ignore[assignment]
        errs = relative_errors(forward(window), reference)
        tried.append((window, errs))
        for h in range(heads):
            if chosen[h] is None and errs[h] <= budget:
                chosen[h], chosen_err[h] = window, errs[h]
        if all(c is not None for c in chosen):
            break
    if any(c is None for c in chosen):
        errs = relative_errors(forward(full), reference)
        tried.append((full, errs))
        for h in range(heads):
            if chosen[h] is None:
                chosen[h], chosen_err[h] = full, errs[h]
    windows = [c for c in chosen if c is not None]
    return WindowSearchResult(windows=windows, errors=chosen_err,
                              keys_per_query=[clamped_keys(w, tile, grid) for w in windows], tried=tried)
