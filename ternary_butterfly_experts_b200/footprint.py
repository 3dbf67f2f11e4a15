"""Stored size of a ButterflyMoE layer against N dense experts.

    python -m ternary_butterfly_experts_b200.footprint [--d D] [--experts N ...] [--angles f32|bf16]

A layer stores one d x d ternary base shared by every expert, its scale, and
per expert the angles of two butterflies, log2(d) stages of d/2 rotations each
(ButterflyMoE technical summary on gist.science, 2.1 and 2.2: memory
O(d^2 + N d log d) against O(N d^2) for N independent experts).  The pages
quote memory figures for d = 512 (2.2 and 4.: 1024 MB against 4.70 MB at 256
experts, 256 MB against 1.9 MB at 64 experts; the arXiv abstract: 80x at 8
experts, 150x at 256).  Their dense baselines count 4 MB per d = 512 expert,
four times a d x d float32 matrix, which the pages do not explain; this tool
counts d x d experts, so its ratios are not the pages' ratios (the figures are
context, not checked values).

Counted per layer:
  base      d^2 weights at 2 bits (the storage of bfmoe_pack_base), and the
            information-theoretic log2(3) = 1.58 bits the pages name;
  alpha     one float32;
  angles    2 N (d/2) log2(d) angles at 4 (float32) or 2 (bf16) bytes;
  dense     N d^2 weights at 4 (float32) or 2 (bf16) bytes.
The runtime's weight tables (cos/sin in kernel order, the bf16 copy of the
base; bfmoe_layer_tables_size) are derived data, rebuilt from the stored
weights, and are listed apart.
"""
from __future__ import annotations

import argparse
import math
from dataclasses import dataclass

MB = 1e6


@dataclass(frozen=True)
class Footprint:
    d: int
    n_experts: int
    angle_bytes: int
    dense_bytes: int
    base_bytes: int          # 2-bit codes, d * ceil(d/16) words of 4 bytes
    base_ideal_bytes: float  # d^2 log2(3) / 8
    alpha_bytes: int
    n_angles: int
    angle_total_bytes: int
    dense_total_bytes: int

    @property
    def stored_bytes(self) -> int:
        return self.base_bytes + self.alpha_bytes + self.angle_total_bytes

    @property
    def ratio(self) -> float:
        return self.dense_total_bytes / self.stored_bytes

    @property
    def per_expert_bytes(self) -> float:
        """Stored bytes per expert, the shared base spread over the N experts."""
        return self.stored_bytes / self.n_experts


def footprint(d: int, n_experts: int, angle_bytes: int = 4, dense_bytes: int = 4) -> Footprint:
    if d < 2 or d & (d - 1):
        raise ValueError("d must be a power of two >= 2")
    if n_experts < 1:
        raise ValueError("n_experts must be >= 1")
    L = d.bit_length() - 1
    words = max(1, (d + 15) // 16)
    n_angles = 2 * n_experts * (d // 2) * L
    return Footprint(
        d=d, n_experts=n_experts, angle_bytes=angle_bytes, dense_bytes=dense_bytes,
        base_bytes=d * words * 4,
        base_ideal_bytes=d * d * math.log2(3) / 8,
        alpha_bytes=4,
        n_angles=n_angles,
        angle_total_bytes=n_angles * angle_bytes,
        dense_total_bytes=n_experts * d * d * dense_bytes,
    )


def table(d: int, experts, angle_bytes: int, dense_bytes: int) -> str:
    rows = ["| N | base (2-bit) | angles | stored | dense N d^2 | dense / stored | per expert |",
            "|---|---|---|---|---|---|---|"]
    for n in experts:
        f = footprint(d, n, angle_bytes, dense_bytes)
        rows.append(f"| {n} | {f.base_bytes / MB:.4f} MB | {f.angle_total_bytes / MB:.4f} MB | "
                    f"{f.stored_bytes / MB:.4f} MB | {f.dense_total_bytes / MB:.1f} MB | {f.ratio:.1f}x | "
                    f"{f.per_expert_bytes / 1e3:.1f} kB |")
    return "\n".join(rows)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--d", type=int, default=512)
    ap.add_argument("--experts", type=int, nargs="*", default=[8, 64, 256])
    ap.add_argument("--angles", choices=["f32", "bf16"], default="f32")
    ap.add_argument("--dense", choices=["f32", "bf16"], default="f32")
    args = ap.parse_args(argv)
    ab = 4 if args.angles == "f32" else 2
    db = 4 if args.dense == "f32" else 2
    print(f"d = {args.d}, angles {args.angles}, dense experts {args.dense} (d x d each)")
    print(table(args.d, args.experts, ab, db))
    return 0


if __name__ == "__main__":
    raise SystemExit(main())
