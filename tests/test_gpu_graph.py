"""The forward path captured into a CUDA graph replays the same kernels as the
eager calls: outputs, masks and skip lists must be bit-identical to the eager
path on the same inputs, also after the inputs change between replays (the
graph reads its static buffers, not the tensors present at capture)."""
import pytest
import torch

import free_block_sparse_predict_b200 as fb
from free_block_sparse_predict_b200.graph import SpargeGraph
from synth import make_qkv

from gpu_common import dev, params_for, to_dev, workload

pytestmark = pytest.mark.gpu


def _eager(p, w, q, k, v):
    perm = None
    if w.grid:
        perm = torch.empty(w.N, dtype=torch.int32, device=dev())
        hws = torch.zeros(fb.sparge_hilbert_workspace_bytes(*w.grid), dtype=torch.uint8,
                          device=dev())
        fb.sparge_hilbert_index(w.N, w.prefix_len, *w.grid, perm, hws)
    return fb.sparge_forward(p, q, k, v, perm=perm)


@pytest.mark.parametrize("name", ["tiny", "image_dit", "llm_32k"])
def test_graph_replay_is_bit_identical_to_eager_calls(name):
    over = {"N": 4160} if name == "llm_32k" else {}
    w, t0 = workload(name, **over)
    p = params_for(w, o_dtype={"f16": torch.float16, "bf16": torch.bfloat16}[w.dtype])
    g = SpargeGraph(p, grid=(w.prefix_len, *w.grid) if w.grid else None, device=dev())
    for seed, t in ((0, t0), (1, make_qkv(w, seed=1))):
        q, k, v = (to_dev(t[x], w.dtype) for x in ("q", "k", "v"))
        o_g = g.run(q, k, v).clone()
        mask_g, cnt_g = g.mask.clone(), g.kv_cnt.clone()
        o_e, mask_e, idx_e, cnt_e = _eager(p, w, q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(mask_g, mask_e), seed
        assert torch.equal(cnt_g, cnt_e), seed
        assert torch.equal(o_g, o_e), seed
        assert fb.sparge_device_status(g.ws) == 0
