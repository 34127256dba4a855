"""Host-side check of the integer block schedule the kernels run
(`csrc/layer_plan.cuh`: blocks, windows, read indices, key segments and
their 128-row tiles, the order blocks are visited in), compiled as host code
and compared exactly with the oracle's definitions. No GPU is used: nvcc
compiles the header's __host__ __device__ functions into a host program."""
import os
import shutil
import subprocess

import numpy as np
import pytest

import oracle as O
import vdn_synth as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_diffusion_hybrid_block_b200", "csrc")

DRIVER = r'''
#include <cstdio>
#include <vector>
#include "layer_plan.cuh"
using namespace vdn;
int main() {
  int F, bf, T;
  if (scanf("%d %d %d", &F, &bf, &T) != 3) return 1;
  std::vector<int32_t> off(F + 1);
  for (int f = 0; f <= F; ++f) scanf("%d", &off[f]);
  const int nb = num_blocks(F, bf);
  printf("nb %d\n", nb);
  for (int b = 0; b < nb; ++b) {
    int w0, w1, i_f, i_b, q0, q1;
    block_window(b, F, bf, w0, w1);
    block_read_indices(b, F, bf, i_f, i_b);
    block_rows(off.data(), F, bf, b, q0, q1);
    const KeySegs s = key_segments(off.data(), F, bf, T, b);
    const int nt = segs_tiles(s);
    printf("block %d %d %d %d %d %d %d %d\n", b, w0, w1, i_f, i_b, q0, q1, nt);
    for (int j = 0; j < nt; ++j) {
      int src, row0, valid;
      segs_tile(s, j, src, row0, valid);
      printf("tile %d %d %d\n", src, row0, valid);
    }
  }
  for (int z = 0; z < nb; ++z) printf("visit %d\n", block_in_visit_order(z, nb));
  return 0;
}
'''


@pytest.fixture(scope="module")
def driver(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    d = tmp_path_factory.mktemp("plan")
    src = d / "plan_driver.cu"
    src.write_text(DRIVER)
    exe = d / "plan_driver"
    subprocess.run([nvcc, "-x", "cu", "-std=c++17", "-I", CSRC, "-o", str(exe), str(src)],
                   check=True, capture_output=True)
    return str(exe)


def run(driver, off, bf, T):
    F = len(off) - 1
    inp = f"{F} {bf} {T}\n" + " ".join(str(int(x)) for x in off) + "\n"
    out = subprocess.run([driver], input=inp, capture_output=True, text=True, check=True).stdout
    blocks, visit, cur = [], [], None
    for line in out.splitlines():
        w = line.split()
        if w[0] == "block":
            cur = dict(b=int(w[1]), window=(int(w[2]), int(w[3])), reads=(int(w[4]), int(w[5])),
                       rows=(int(w[6]), int(w[7])), ntiles=int(w[8]), tiles=[])
            blocks.append(cur)
        elif w[0] == "tile":
            cur["tiles"].append((int(w[1]), int(w[2]), int(w[3])))
        elif w[0] == "visit":
            visit.append(int(w[1]))
    return blocks, visit


def _layouts():
    rng = np.random.default_rng(3)
    return [
        ("pages-scale", S.frame_offsets(S.frame_sizes(S.CONFIGS["pages-scale"])), 5, 256),
        ("vda-stress", S.frame_offsets(S.frame_sizes(S.CONFIGS["vda-stress"])), 5, 128),
        ("zero-frames", S.frame_offsets([40, 30, 0, 25, 0, 60, 1, 20, 33, 0, 17, 9]), 5, 6),
        ("F2", S.frame_offsets([70, 9]), 5, 5),
        ("no-text", S.frame_offsets([50] * 13), 5, 0),
        ("bf3", S.frame_offsets([130] * 14), 3, 40),
        ("F4096", S.frame_offsets(rng.integers(0, 4, size=4096)), 5, 4),
        ("big-frames", S.frame_offsets([1792] * 20), 5, 512),
        ("bf1", S.frame_offsets([37, 0, 5, 129, 64, 2, 90, 11, 40]), 1, 7),
        ("bf7", S.frame_offsets([110] * 30), 7, 33),
        ("bf-larger-than-F", S.frame_offsets([20, 30, 0, 9]), 6, 3),
    ]


@pytest.mark.parametrize("name,off,bf,T", _layouts(), ids=[x[0] for x in _layouts()])
def test_schedule_matches_oracle(driver, name, off, bf, T):
    off = np.asarray(off, np.int64)
    F = len(off) - 1
    blocks, visit = run(driver, off, bf, T)
    nb = O.num_blocks(F, bf)
    assert len(blocks) == nb
    for blk in blocks:
        b = blk["b"]
        assert blk["window"] == O.window(b, F, bf)
        assert blk["reads"] == O.read_indices(b, F, bf)
        assert blk["rows"] == (int(off[bf * b]), int(off[min(bf * b + bf, F)]))
        # the tiles cover exactly the allowed keys, each once
        want = {(1, r) for r in range(T)}
        for f in O.softmax_key_frames(b, F, bf):
            want |= {(0, r) for r in range(int(off[f]), int(off[f + 1]))}
        got = []
        for src, row0, valid in blk["tiles"]:
            assert 1 <= valid <= 128, (b, src, row0, valid)
            got += [(src, r) for r in range(row0, row0 + valid)]
        assert len(got) == len(set(got)), "a key row is visited twice"
        assert set(got) == want
        assert blk["ntiles"] == len(blk["tiles"])
        # only the last tile of a key segment (text, then at most three merged
        # frame ranges) is partial
        assert sum(1 for _, _, v in blk["tiles"] if v < 128) <= 4
    # blocks are visited once each, interior blocks (full windows) first
    assert sorted(visit) == list(range(nb))
    if nb >= 3:
        assert set(visit[:nb - 2]) == set(range(1, nb - 1))
