"""Single-tile work items with the tile-0 softmax held back.

A node with an odd number of query tiles ends in a pair that holds one tile.
The second MMA thread skips such an item, so its next S must wait until the
S buffer's previous owner, the single-tile item's last S, has been loaded;
an S issued earlier would overwrite it. This test builds a copy of the
attention kernel whose tile-0 softmax holds the last S of every single-tile
item for 4 us before loading it, which keeps that window open, and runs a
round whose items are half single-tile (tests/single_tile_round.py). The
copy must finish without a stopped wait, give the in-tree kernel's output bit
for bit, and match the float64 oracle (max-abs 1e-2, rel-L2 5e-3 per node).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

import single_tile_round as rnd
from wave_testlib import assert_close, oracle_outputs, torch_to_f64

pytestmark = pytest.mark.gpu

# The statement that loads the S row in the softmax; the hold goes before it.
ANCHOR = "        tmem_ld128_wait(tS, *reinterpret_cast<uint32_t(*)[128]>(sv));\n"
HOLD = ("        if (wq == 0 && !w.two && t + 1 == w.n_pages) {  // test build: hold this load\n"
        "          const uint64_t t_hold = globaltimer_ns();\n"
        "          while (globaltimer_ns() - t_hold < 4000) {\n"
        "          }\n"
        "        }\n")


def test_held_single_tile_items(cuda_lib, tmp_path):
    from block_causal_attention_wave_b200 import build

    text = open(os.path.join(build.PKG, "csrc", "wave_attn.cu")).read()
    assert text.count(ANCHOR) == 1, "the S-row load statement moved: update the anchor"
    held_src = tmp_path / "wave_attn.cu"
    held_src.write_text(text.replace(ANCHOR, HOLD + ANCHOR))
    # Built in-tree (the package's git-ignored _build folder), like the library itself.
    os.makedirs(os.path.join(build.PKG, "_build"), exist_ok=True)
    lib = build.build(out=os.path.join(build.PKG, "_build", "libwave_held.so"),
                      replace={"wave_attn.cu": str(held_src)})

    out = tmp_path / "held.npy"
    r = subprocess.run([sys.executable, rnd.__file__, str(out)],
                       env=dict(os.environ, WAVE_LIBRARY=lib),
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    held = np.load(out)

    active, inp, o = rnd.run(cuda_lib)
    assert np.array_equal(held, rnd.output_bits(o)), "held build differs from the in-tree kernel"

    wl = rnd.WL
    want = oracle_outputs(inp, active, rnd.POLICY)
    got = torch_to_f64(o).reshape(len(active), wl.tokens, wl.heads, wl.head_dim)
    for i, n in enumerate(active):
        assert_close(got[i], want[n], f"{wl.name} node {n}")
