"""Branch-specific placement of the hybrid layer on two ranks.

The pages run the softmax branch and the linear (VDA) branch of the layer on
different devices, instead of splitting heads or sequence across devices
["VDN-MiniMax-H3" (openi.cn), 主要功能 item 5; "VDN-MiniMax-H3 - OpenVDN's
Open-Source Video Generation Acceleration Solution" (nav.superapi.store),
Main Features, Branch-Specific Parallelism]. Here, one process per GPU:

* rank LINEAR_RANK runs the linear branch up to the packed read states
  (``vdn_vda_read_images``: Grams, inverses, both scans, R_b as one 32 KB
  bf16 tile per (block, head)) and sends the tiles to the softmax rank;
* rank SOFTMAX_RANK receives them into its own memory, then runs the softmax
  branch with the readout, RMSNorm and gated merge fused in its epilogue
  (``vdn_bsa_merge_fwd``) and holds the layer output.

The exchange is the only collective step (nb * H * 32 KB: 3 MB for 24 heads
and 4 blocks), a point-to-point send / receive over the process group (NCCL
over NVLink between GPUs). The softmax rank's kernel is launched after the
receive on the same stream, so no kernel waits on another rank's kernel.
Both ranks hold the layer's inputs. The compute steps are passed in as a
``backend`` object so that the exchange can be exercised without a GPU.
"""
from __future__ import annotations

SOFTMAX_RANK = 0
LINEAR_RANK = 1


class DeviceBackend:
    """The two compute steps on this rank's GPU, through the C ABI."""

    def __init__(self, binding_module=None):
        if binding_module is None:
            from . import binding as binding_module
        self.B = binding_module

    def read_images(self, shape, inp, rimg, workspace):
        self.B.vdn_vda_read_images(shape, inp["k"], inp["v"], inp["kt"], inp["vt"], rimg,
                                   workspace)

    def merge(self, shape, inp, rimg, out, workspace):
        self.B.vdn_bsa_merge_fwd(shape, inp["q"], inp["k"], inp["v"], inp["kt"], inp["vt"],
                                 inp["g_s"], inp["g_l"], inp["rms_w"], rimg, out, workspace)


def branch_parallel_forward(dist, shape, inp: dict, rimg, out, workspace, backend=None):
    """One layer forward with the branches on two ranks of the default
    process group (world size 2). Every rank calls it with the same shape;
    ``rimg`` is this rank's buffer for the read-state tiles, ``out`` and
    ``workspace`` this rank's output and workspace. Returns ``out`` on the
    softmax rank (written) and None on the linear rank."""
    backend = backend or DeviceBackend()
    if dist.get_world_size() != 2:
        raise ValueError("branch-specific placement runs on exactly two ranks")
    rank = dist.get_rank()
    if rank == LINEAR_RANK:
        backend.read_images(shape, inp, rimg, workspace)
        dist.send(rimg, dst=SOFTMAX_RANK)
        return None
    dist.recv(rimg, src=LINEAR_RANK)
    backend.merge(shape, inp, rimg, out, workspace)
    return out
