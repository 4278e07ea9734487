"""Seeded synthetic inputs for block-sparse attention driven by a per-input mask.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests.  It holds none of the method's arithmetic: it only draws random
numbers, rounds them to bf16, and describes the workloads (shapes, token
segments, head masks, density budgets).

Recipe:
  rng = numpy.random.default_rng([seed, layer, tensor_id]) with tensor_id
  Q=0, K=1, V=2, P=3, head-mask=4.
  V ~ N(0, 1).
  Q = 0.5*N(0,1) + phi(pos) @ P_h,  K = 0.5*N(0,1) + phi(pos) @ P_h, where
  P_h in R^{8 x d} has N(0,1)/sqrt(8) entries (same P_h for Q and K, so
  Q.K^T carries a cos(w*delta) locality term).  Text and padding tokens have
  phi = 0.  2D grids use [sin, cos](pi*y/Gy), [sin, cos](2*pi*y/Gy),
  [sin, cos](pi*x/Gx), [sin, cos](2*pi*x/Gx); 3D (t, y, x) grids use
  [sin, cos](pi*t/T), [sin, cos](2*pi*t/T), [sin, cos](pi*y/G),
  [sin, cos](pi*x/G).  The "plain" generator draws Q, K, V ~ N(0, 1).
  All values are rounded to bf16 by round-to-nearest-even from float32.
"""
from .synth import (SEG_TEXT, SEG_PAD, SEG_IMAGE, SEG_OTHER, Workload, WORKLOADS,
                    bf16_bits_from_f32, bf16_bits_to_f32, make_qkv, head_mask_for_layer,
                    make_workload)

__all__ = ["SEG_TEXT", "SEG_PAD", "SEG_IMAGE", "SEG_OTHER", "Workload", "WORKLOADS",
           "bf16_bits_from_f32", "bf16_bits_to_f32", "make_qkv", "head_mask_for_layer",
           "make_workload"]
