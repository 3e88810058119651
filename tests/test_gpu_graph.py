"""fr_beam_reset, fr_beam_step and fr_beam_finalize allocate nothing and
never synchronise, so a whole decode can be captured into one CUDA graph and
replayed; the replay must give bit-identical results to the eager decode."""
import numpy as np
import pytest
import torch

from trie_constrained_beam_fr_b200 import fr, synth

from frlib import GpuBeam

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_decode_captured_in_a_cuda_graph(name):
    w = synth.WORKLOADS["tiny"] if name == "tiny" else synth.Workload(
        "mid", B=4, K=64, depth=3, C=64, V=20000, sid_base=1000, n_items=20000, dtype="bf16", seed=2, catalog_seed=2)
    sids = synth.workload_catalog(w)
    gpu = GpuBeam(w, sids)
    try:
        # eager decode; keep each step's logits in its own buffer
        bufs = []
        fr.fr_beam_reset(gpu.beam)
        for t in range(w.depth):
            gpu.gen_logits(t)
            bufs.append(gpu.logits.clone())
            fr.fr_beam_step(gpu.beam, bufs[-1], ld=gpu.ld)
        eager = gpu.finalize()
        out_sids = torch.empty((w.B, w.K, w.depth), dtype=torch.int32, device="cuda")
        out_scores = torch.empty((w.B, w.K), dtype=torch.float32, device="cuda")
        out_items = torch.empty((w.B, w.K), dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fr.fr_beam_reset(gpu.beam)
            for t in range(w.depth):
                fr.fr_beam_step(gpu.beam, bufs[t], ld=gpu.ld)
            fr.fr_beam_finalize(gpu.beam, out_sids, out_scores, out_items)
        for _ in range(2):
            out_scores.fill_(0)
            g.replay()
            torch.cuda.synchronize()
            assert fr.fr_beam_status(gpu.beam) == fr.FR_OK
            np.testing.assert_array_equal(out_sids.cpu().numpy(), eager[0])
            np.testing.assert_array_equal(out_scores.cpu().numpy().view(np.uint32), eager[1].view(np.uint32))
            np.testing.assert_array_equal(out_items.cpu().numpy(), eager[2])
        del g
    finally:
        gpu.close()


def test_lmhead_decode_captured_in_a_cuda_graph():
    """The lm_head path (fused tensor-core lm_head + step from the SID slice)
    in one graph: its TMA descriptors are encoded when the launch is captured,
    so replays read the same buffers and give the eager results bit for bit."""
    w = synth.Workload("lm_graph", B=3, K=32, depth=3, C=16, V=1000, sid_base=100, n_items=2000, dtype="bf16",
                       seed=31, catalog_seed=31)
    d = 128
    sids = synth.workload_catalog(w)
    span = w.depth * w.C
    gpu = GpuBeam(w, sids)
    Wd = torch.from_numpy(synth.lm_head_weight(7, w.V, d)).to(torch.bfloat16).cuda()
    g = torch.Generator(device="cuda").manual_seed(5)
    hidden = [torch.randn(w.B, w.K, d, device="cuda", generator=g).to(torch.bfloat16) for _ in range(w.depth)]
    lm = fr.fr_lmhead_init(Wd, max_rows=w.B * w.K, sid_base=w.sid_base, sid_span=span)
    lse = torch.empty(w.B * w.K, device="cuda")
    sl = torch.empty(w.B * w.K, span, device="cuda")
    out = (torch.empty((w.B, w.K, w.depth), dtype=torch.int32, device="cuda"),
           torch.empty((w.B, w.K), dtype=torch.float32, device="cuda"),
           torch.empty((w.B, w.K), dtype=torch.int32, device="cuda"))

    def decode():
        fr.fr_beam_reset(gpu.beam)
        for t in range(w.depth):
            rows = w.B if t == 0 else w.B * w.K
            h = hidden[t][:, 0, :] if t == 0 else hidden[t].view(rows, d)
            fr.fr_lmhead_run(lm, h, lse[:rows], sl[:rows])
            fr.fr_beam_step_lse(gpu.beam, lse[:rows], sl[:rows], 1 if t == 0 else w.K)
        fr.fr_beam_finalize(gpu.beam, *out)

    try:
        decode()
        torch.cuda.synchronize()
        assert fr.fr_lmhead_status(lm) == fr.FR_OK and fr.fr_beam_status(gpu.beam) == fr.FR_OK
        eager = [x.cpu().numpy().copy() for x in out]
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            decode()
        for _ in range(2):
            out[1].fill_(0)
            graph.replay()
            torch.cuda.synchronize()
            assert fr.fr_lmhead_status(lm) == fr.FR_OK and fr.fr_beam_status(gpu.beam) == fr.FR_OK
            np.testing.assert_array_equal(out[0].cpu().numpy(), eager[0])
            np.testing.assert_array_equal(out[1].cpu().numpy().view(np.uint32), eager[1].view(np.uint32))
            np.testing.assert_array_equal(out[2].cpu().numpy(), eager[2])
        del graph
    finally:
        fr.fr_lmhead_destroy(lm)
        gpu.close()
