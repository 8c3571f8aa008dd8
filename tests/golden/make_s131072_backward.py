"""Writes tests/golden/s131072_d8_seed4.npz: fp64-oracle values of the 7B-shaped
layer at S=131072, D=8, seed 4 (h=4096, 32 heads x 128, FFN 16384), for the
GPU parity test at that size.

It calls only ``oracle`` and ``synth_inputs``.  The oracle result is the
unsharded layer in global token order (the folded layer equals it: the folding
identity pinned in tests/test_oracle_pins.py); the stored rows are named both
by their rank-major (zigzag, D=8) index and by their global position.

Stored (fp32 values, int64 indices):
  rows, pos        the 512 seeded sample rows (rank-major index, global position),
                   rows 0 and S-1 included (synth_inputs.sample_rows);
  z, dx            those rows of the layer output and of the input gradient;
  dg1, dg2         both gain gradients, every element;
  {dwqkv,dwo,dw1,dw2}_idx / _val
                   65,536 distinct flat indices per weight gradient, drawn with
                   np.random.default_rng(seed + 2000), and the values there;
  input_sha256     hash of the bf16 bit patterns of x, Wqkv, Wo, W1, W2, dY;
  meta             the shape and seed, as text.

Run once on a host with ~48 GB of free RAM and ~40 GB of free disk under
$TMPDIR (about two hours on 8 cores):
    python tests/golden/make_s131072_backward.py [workers]
"""

from __future__ import annotations

import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from synth_inputs import WORKLOADS, bits_to_f32, input_hash, make_layer_inputs, sample_rows  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "s131072_d8_seed4.npz")
N_W_SAMPLES = 65536


def weight_sample(shape, seed):
    rng = np.random.default_rng(seed + 2000)
    out = {}
    for name, shp in shape.items():
        out[name] = np.sort(rng.choice(int(np.prod(shp)), size=N_W_SAMPLES, replace=False)).astype(np.int64)
    return out


def main(workers: int):
    shape, seed = WORKLOADS["7b_s128k"]
    t0 = time.time()
    log = lambda m: print(f"[{time.time() - t0:8.1f} s] {m}", flush=True)
    inp = make_layer_inputs(shape, seed)
    digest = input_hash(inp)
    log(f"inputs drawn, sha256 {digest}")
    w = {k: bits_to_f32(inp[k]).astype(np.float64) for k in ("wqkv", "wo", "w1", "w2")}
    w["g1"] = inp["g1"].astype(np.float64)
    w["g2"] = inp["g2"].astype(np.float64)
    x = bits_to_f32(inp["x"]).astype(np.float64)
    dz = bits_to_f32(inp["dy"]).astype(np.float64)
    del inp
    res = O.layer_forward_backward_blocked(x, w, dz, shape.heads, row_block=4096, workers=workers, log=log)
    del x, dz
    rows = sample_rows(shape.S, 512, seed)
    pos = O.zigzag_map(shape.S, shape.D).ravel()[rows]
    h, F = shape.h, shape.ffn
    wshape = {"dwqkv": (3 * h, h), "dwo": (h, h), "dw1": (F, h), "dw2": (h, F)}
    idx = weight_sample(wshape, seed)
    out = dict(rows=rows.astype(np.int64), pos=pos.astype(np.int64),
               z=res["z"][pos].astype(np.float32), dx=res["dx"][pos].astype(np.float32),
               dg1=res["dg1"].astype(np.float32), dg2=res["dg2"].astype(np.float32),
               input_sha256=np.array(digest),
               meta=np.array(f"h={h} heads={shape.heads} ffn={F} S={shape.S} D={shape.D} seed={seed}"))
    for name in wshape:
        out[name + "_idx"] = idx[name]
        out[name + "_val"] = res[name].ravel()[idx[name]].astype(np.float32)
    np.savez_compressed(OUT, **out)
    log(f"wrote {OUT}")


if __name__ == "__main__":
    main(int(sys.argv[1]) if len(sys.argv) > 1 else os.cpu_count())
