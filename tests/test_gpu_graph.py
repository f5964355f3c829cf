"""The whole hot-path step captured into a CUDA graph: every stage is a
stream-ordered C-ABI call (the planner's fork onto the library's side stream and
its join included), so capture works and replays give the eager results bit for
bit (the deterministic backward)."""
import pytest
import torch

import block_sparse_attention_map_b200 as bsa
from block_sparse_attention_map_b200.workloads import make_workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["window", "document"])
def test_step_captured_in_a_graph_replays_the_eager_results(name):
    wl = make_workload(name, device="cuda", small=True)
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")

    def step():
        st.plan_and_bound()
        st.forward()
        st.preprocess(wl.dO)
        st.backward_main(wl.dO)
        st.convert()

    step()  # eager (also creates the library's side stream before any capture)
    torch.cuda.synchronize()
    assert st.ws.status() == 0
    ref = [t.clone() for t in (st.out, st.lse, st.dq, st.dk, st.dv)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        step()
    for _ in range(2):
        for t in (st.out, st.lse, st.dq, st.dk, st.dv):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert st.ws.status() == 0
        got = (st.out, st.lse, st.dq, st.dk, st.dv)
        assert all(torch.equal(a, b) for a, b in zip(ref, got))


# header words of the persistent kernels' work tickets and their exit counts
# (csrc/internal.h: the forward's unit ticket 2, the backward's column ticket 3,
# their exit counters 14 and 15)
_TICKET_WORDS = (2, 3, 14, 15)


@pytest.mark.parametrize("name", ["window", "packed"])
def test_work_tickets_return_to_zero_after_every_launch(name):
    """The forward and the backward draw work from ticket words in the
    workspace header, and the last CTA of each launch puts them back to zero
    (no memset precedes the launch).  Launch after launch on one workspace,
    without a new plan, eager and replayed from a graph: the words read zero
    after every step and every step's results are bit-identical."""
    wl = make_workload(name, device="cuda", small=True)
    st = bsa.Stages(wl.q, wl.k, wl.v, wl.mask, softmax_mode="fixed_m", order="desc")
    st.plan_and_bound()

    def step():
        st.forward()
        st.preprocess(wl.dO)
        st.backward_main(wl.dO)
        st.convert()

    ref = None
    for it in range(3):
        step()
        torch.cuda.synchronize()
        assert st.ws.status() == 0
        hdr = st.ws.header().cpu()
        assert all(int(hdr[w]) == 0 for w in _TICKET_WORDS), hdr[list(_TICKET_WORDS)]
        got = [t.clone() for t in (st.out, st.lse, st.dq, st.dk, st.dv)]
        if ref is None:
            ref = got
        else:
            assert all(torch.equal(a, b) for a, b in zip(ref, got))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        step()
    for _ in range(3):
        for t in (st.out, st.lse, st.dq, st.dk, st.dv):
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert st.ws.status() == 0
        hdr = st.ws.header().cpu()
        assert all(int(hdr[w]) == 0 for w in _TICKET_WORDS), hdr[list(_TICKET_WORDS)]
        got = (st.out, st.lse, st.dq, st.dk, st.dv)
        assert all(torch.equal(a, b) for a, b in zip(ref, got))
