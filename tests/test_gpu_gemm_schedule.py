"""GPU parity of the fused dequant GEMMs under their persistent schedule, where
the K-steps of the tiles left over after the full waves are shared between
CTAs: a CTA that computes part of a tile leaves an fp32 partial in the
workspace, and the CTA holding the tile's first K-step adds the partials and
writes the output.

`qlora_gemm_set_ctas` caps the grid (CTA pairs on 512 x 256 tiles) so that
small layers take the same paths a 74-pair launch takes on the large ones:
tiles split two to four ways, whole tiles followed by split ones, adapter
K-steps inside a split, ragged M.
Each case is compared with the float64 oracle (relative Frobenius <= 1e-2,
max-abs <= 2e-2 of max |ref|) on every output.  The full-size layers of
test_gpu_linear run the uncapped grid: at M = 4096 the 4096 x 4096 layer has
74 whole pair tiles and 54 split ones.  With fewer tiles than pairs the tiles are
split only when that saves more than the extra work item costs: at M = 2048 (the
stack) the 4096 x 4096 layers run their 64 tiles whole, the 11008-deep down
projection splits its 64 tiles over the 74 pairs."""

import pytest
import torch

import quantized_rank_fine_b200 as q
from tests.helpers import assert_close, full_check, layer_on_gpu, require_gpu, run_fwd_bwd

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _gpu():
    require_gpu()
    yield
    q.qlora_gemm_set_ctas(0)


def _align256(n):
    return (n + 255) // 256 * 256


# the workspace prefix: status word (256 B), then the GEMM's 256 counters
COUNTERS = slice(256, 1280)


def _partials_offset(op, M, r):
    """Byte offset of the GEMM's partial tiles in a workspace."""
    mr = _align256(M * r * 2)
    return 1280 + mr * (1 if op == q.QLORA_OP_FWD else 2)


# (M, in, out, r, CTAs): the forward GEMM has N = out, K = in; dX has N = in, K = out.
# The GEMM runs CTA pairs on 512 x 256 tiles, so CTAs / 2 pairs share the work.
CASES = [
    (600, 2048, 768, 24, 24),   # fwd: 6 tiles, all split over 12 pairs; dX: 16 tiles, all split over 12 pairs
    (256, 4096, 256, 16, 8),    # fwd: one tile's 65 K-steps over 4 pairs (the owner adds 3 partials)
    (256, 256, 4096, 72, 8),    # dX: one tile over 4 pairs, its two adapter K-steps in the last share
    (1100, 2048, 1536, 40, 10), # fwd and dX: whole tiles, then split ones; M ragged (76 rows in the last tile)
    (777, 1024, 1280, 64, 6),   # fwd: 6 whole tiles, then 4 split over 3 pairs; M ragged
    (1500, 1024, 1280, 64, 10), # dX: 5 whole tiles, then 7 split over 5 pairs; M ragged
    (9000, 64, 128, 64, 8),     # fwd and dX: 18 whole tiles of 2 or 3 K-steps (one adapter step) over 4
                                # pairs, four or five items a pair back to back; M ragged
]


@pytest.mark.parametrize("M,n_in,n_out,r,ctas", CASES)
def test_split_schedule_matches_oracle(M, n_in, n_out, r, ctas):
    q.qlora_gemm_set_ctas(ctas)
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="sched")
    full_check(t, w, run_fwd_bwd(t, w))


def test_split_schedule_deterministic_counters_cleared_and_graph():
    """Repeated calls give identical bytes (the partials are added in a fixed
    order), the counters are back at zero after each call, and CUDA-graph
    replays of the same calls reproduce the eager results."""
    M, n_in, n_out, r = 1100, 2048, 1536, 40
    q.qlora_gemm_set_ctas(10)
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="sched")
    ws = q.Workspace()
    Y, V = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(ws.buf[COUNTERS]).item() == 0, "counters not cleared by the forward"
    first = run_fwd_bwd(t, w, ws)
    assert torch.count_nonzero(ws.buf[COUNTERS]).item() == 0, "counters not cleared by the backward"
    assert torch.equal(Y, first["Y"])
    again = run_fwd_bwd(t, w, ws)
    for k in ("Y", "dX", "dA", "dB"):
        assert torch.equal(first[k], again[k]), k

    Y = torch.empty_like(first["Y"])
    V = torch.empty_like(first["V"])
    dX = torch.empty_like(first["dX"])
    dA = torch.empty_like(first["dA"])
    dB = torch.empty_like(first["dB"])
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws, Y=Y, V=V)
            q.qlora_linear_bwd(w, t["X"], V, t["dY"], t["A"], t["B"], ws, dX=dX, dA=dA, dB=dB)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(3):
        Y.zero_()
        dX.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(Y, first["Y"]) and torch.equal(dX, first["dX"])
        assert torch.equal(dA, first["dA"]) and torch.equal(dB, first["dB"])
    del graph
    assert ws.status() == 0


class _CappedWorkspace(q.Workspace):
    """A workspace that never grows past `cap` bytes."""

    def __init__(self, cap):
        super().__init__()
        self.cap = cap

    def get(self, nbytes, stream=None):
        return super().get(min(nbytes, self.cap), stream)


def test_workspace_without_split_region_keeps_tiles_whole():
    """A workspace that ends before the split region is accepted; the GEMMs then
    keep every tile whole.  Both schedules match the oracle, and they differ
    only by the order of fp32 additions."""
    M, n_in, n_out, r = 1100, 2048, 1536, 40
    q.qlora_gemm_set_ctas(10)
    t, w = layer_on_gpu(n_in, n_out, M, r, tag="sched")
    split = run_fwd_bwd(t, w, q.Workspace())
    full = q.qlora_workspace_bytes(q.QLORA_OP_BWD, M, n_in, n_out, r)
    cap = _partials_offset(q.QLORA_OP_BWD, M, r)
    assert full > cap, "this case must use a split region"
    whole = run_fwd_bwd(t, w, _CappedWorkspace(cap))
    full_check(t, w, whole)
    for k in ("Y", "dX"):
        # at most one bf16 rounding step apart (2^-7 relative) where the fp32 sums straddle a boundary
        assert_close(whole[k], split[k].double().cpu().numpy(), f"{k} whole vs split", rel_fro=2e-3, max_abs=1e-2)
    assert torch.equal(whole["dA"], split["dA"]) and torch.equal(whole["dB"], split["dB"])


@pytest.mark.parametrize("n_out", [128, 192])
def test_partial_column_tile_repeated(n_out):
    """A pair tile wider than the output: each warp stores a prefix of its 32-column
    blocks and skips the rest, and the staging buffers of the stored blocks must not
    be touched again until their TMA stores have read them.  Short items (two K-steps)
    back to back make a late store likely; ten forwards must give the same bytes,
    and the first matches the oracle."""
    t, w = layer_on_gpu(64, n_out, 131062, 64, tag="partcol")   # 256 tiles: 3-4 items a pair
    ws = q.Workspace()
    first = run_fwd_bwd(t, w, ws)
    full_check(t, w, first)
    for _ in range(10):
        Y, _ = q.qlora_linear_fwd(w, t["X"], t["A"], t["B"], ws)
        torch.cuda.synchronize()
        assert torch.equal(Y, first["Y"])
