"""Branch-specific placement (two ranks): the exchange logic on CPU with two
gloo ranks, and a failing linear rank detected by the softmax rank through
the process group's timeout (no GPU involved).

The CPU backend stands in for the two device steps with the oracle: the
linear rank computes each head's read states R_b, the softmax rank combines
the received R_b with the oracle's softmax branch and gated merge. The
softmax rank's output must equal the oracle's whole layer, which holds only
if the read states crossed the process group intact and in order. The GPU
path of the same split (vdn_vda_read_images + vdn_bsa_merge_fwd equals
vdn_hybrid_attn_fwd bit for bit) is tested on one GPU in test_gpu_parity.py."""
import datetime
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleBackend:
    """CPU stand-in for the two device steps (float64 read states)."""

    def read_images(self, shape, inp, rimg, workspace):
        import oracle as O
        H = inp["H"]
        R = np.stack([O.vda_states_head(inp["k"], inp["v"], inp["kt"], inp["vt"], inp["off"], h,
                                        inp["lam"], inp["block_frames"])["R"]
                      for h in range(H)], axis=1)               # [nb, H, d, d]
        rimg.copy_(torch.from_numpy(R))

    def merge(self, shape, inp, rimg, out, workspace):
        import oracle as O
        R = rimg.numpy()
        off = np.asarray(inp["off"])
        fid = np.repeat(np.arange(inp["F"]), np.diff(off))
        blk = fid // inp["block_frames"]
        for h in range(inp["H"]):
            o_soft = O.softmax_branch_head(inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                           off, h, inp["block_frames"])
            q = inp["q"][:, h].astype(np.float64)
            o_lin = np.einsum("nd,nde->ne", q, R[blk, h])
            out[:, h] = torch.from_numpy(O.gate_merge(o_soft, o_lin, inp["g_s"][:, h],
                                                      inp["g_l"][:, h], inp["rms_w"][h],
                                                      inp["eps"]))


def _inputs():
    import vdn_synth as S
    return S.make_inputs_from(16, [5] * 16, 4, 2, 8, dtype="f32", seed=3)


def _rank(rank, port, q, fail_linear):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist

    import oracle as O
    from video_diffusion_hybrid_block_b200.branch_parallel import branch_parallel_forward
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=2,
                            timeout=datetime.timedelta(seconds=10))
    try:
        inp = _inputs()
        nb = O.num_blocks(inp["F"], inp["block_frames"])
        rimg = torch.zeros((nb, inp["H"], inp["d"], inp["d"]), dtype=torch.float64)
        out = torch.zeros((inp["N"], inp["H"], inp["d"]), dtype=torch.float64)
        if fail_linear and rank == 1:
            raise RuntimeError("linear rank failed before sending")
        try:
            got = branch_parallel_forward(dist, None, inp, rimg, out, None,
                                          backend=OracleBackend())
        except RuntimeError as e:  # the receive gave up: the other rank is gone
            q.put((rank, "error", str(e)[:80]))
            return
        if rank == 0:
            ref = np.stack([O.layer_head(inp, h)["out"] for h in range(inp["H"])], axis=1)
            q.put((rank, "ok", float(np.abs(got.numpy() - ref).max())))
        else:
            q.put((rank, "ok", got))
    except RuntimeError as e:
        q.put((rank, "raised", str(e)[:80]))
    finally:
        if not (fail_linear and rank == 1):
            try:
                dist.destroy_process_group()
            except Exception:  # noqa: BLE001
                pass


def _run(fail_linear):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + (os.getpid() % 1000) + (7 if fail_linear else 0)
    procs = [ctx.Process(target=_rank, args=(r, port, q, fail_linear)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
    return dict((r, (status, val)) for r, status, val in (q.get(timeout=10) for _ in range(2)))


def test_two_gloo_ranks_compose_the_layer():
    res = _run(fail_linear=False)
    assert res[1] == ("ok", None)                 # the linear rank holds no output
    assert res[0][0] == "ok" and res[0][1] < 1e-12, res[0]


def test_softmax_rank_detects_a_failed_linear_rank():
    # the linear rank raises before its send; the softmax rank's receive must
    # end with an error (process-group timeout or closed connection), not hang
    res = _run(fail_linear=True)
    assert res[1][0] == "raised"
    assert res[0][0] == "error", res[0]


def test_rejects_other_world_sizes():
    sys.path.insert(0, ROOT)
    from video_diffusion_hybrid_block_b200.branch_parallel import branch_parallel_forward

    class One:
        def get_world_size(self):
            return 1

    with pytest.raises(ValueError):
        branch_parallel_forward(One(), None, {}, None, None, None, backend=OracleBackend())
