"""The layer loop's host logic on CPU: which layers a step acquires, prefetches
and releases, in which order, through an S-slot pool.

The stack's sweeps run unchanged; the library calls they make are replaced by
fakes: a pool that follows the slot rules lsnf4.h states for layer_pool_*
(a copy takes the least recently released slot that is neither acquired nor
holding a prefetched, not yet acquired layer, else LSN_ERR_STATE; a prefetch
of a resident layer keeps it until it is acquired), and compute calls that
only return success.  Checked: no call ever finds the pool without a free
slot, every acquire is released, the layers come in sweep order, and a step
copies 2L - S layers the first time and 2L - 2S after that."""
import pytest
import torch

from layer_streamed_nf4_b200 import lsnf4, synth
from layer_streamed_nf4_b200.stack import Stack, layer_layout


class FakePool:
    def __init__(self, n_slots):
        self.layer = [-1] * n_slots
        self.refs = [0] * n_slots
        self.pending = [False] * n_slots
        self.last_release = [0] * n_slots
        self.tick = 0
        self.copies = 0
        self.held = {}
        self.acquired = []

    def _find(self, l):
        return self.layer.index(l) if l in self.layer else -1

    def _copy(self, l):
        best = -1
        for s in range(len(self.layer)):
            if self.refs[s] > 0 or self.pending[s]:
                continue
            if best < 0 or self.last_release[s] < self.last_release[best] or (
                    self.last_release[s] == self.last_release[best] and self.layer[s] < 0 <= self.layer[best]):
                best = s
        if best < 0:
            raise lsnf4.LsnError(lsnf4.LSN_ERR_STATE, "fake layer pool", "no free slot")
        self.layer[best] = l
        self.pending[best] = True
        self.copies += 1
        return best

    def prefetch(self, pool, l):
        s = self._find(l)
        if s >= 0:
            if self.refs[s] == 0:
                self.pending[s] = True
            return
        self._copy(l)

    def acquire(self, pool, l, stream):
        s = self._find(l)
        if s < 0:
            s = self._copy(l)
        self.pending[s] = False
        self.refs[s] += 1
        self.held.setdefault(l, []).append(s)
        self.acquired.append(l)
        return (s + 1) << 20

    def release(self, pool, l, stream):
        s = self.held[l].pop()
        self.refs[s] -= 1
        self.tick += 1
        self.last_release[s] = self.tick


class FakeStream:
    cuda_stream = 0

    def wait_event(self, ev):
        pass


class FakeEvent:
    def record(self, stream=None):
        pass


class FakeLib:
    """The compute entry points the sweeps call directly: success, nothing done."""

    def __getattr__(self, name):
        return lambda *args: 0


def _cpu_stack(monkeypatch, L, S, ahead, api="layer"):
    cfg = synth.StackConfig("tiny", L, 64, 64, 128, 4, 8, 16.0, "nf4")
    st = Stack.__new__(Stack)
    st.cfg, st.mode, st.seed = cfg, "streamed", 7
    st.api, st.grouped, st.shared_inputs = api, False, False
    st.L, st.T, st.r, st.scale = L, cfg.tokens, cfg.rank, cfg.alpha / cfg.rank
    st.nf4, st.kind = True, lsnf4.LSN_BASE_NF4
    st.dev = torch.device("cpu")
    st.stream = FakeStream()
    st.keep_outputs = False
    st.n_lanes, st.lanes, st._fork, st._join = 1, [st.stream], [FakeEvent()], [FakeEvent()]
    st.proj, st.layer_bytes, st.const_bytes = layer_layout(cfg, True)
    st.consts = torch.zeros((L, st.const_bytes), dtype=torch.uint8)
    st._calls, st._distinct, st._ahead_opt, st.ahead_blocks_per_sm = {}, True, ahead, 8
    st.ahead = st._ahead_for("streamed")
    st._wbuf = [torch.empty(sum(p.N * p.K for p in st.proj), dtype=torch.bfloat16) for _ in range(2)]
    st._woff, o = [], 0
    for p in st.proj:
        st._woff.append(o)
        o += p.N * p.K
    st._prep = FakeStream()
    st._ev_ready = [FakeEvent(), FakeEvent()]
    st._ev_done = [FakeEvent(), FakeEvent()]
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    st._build_tensors(True)
    pool = FakePool(S)
    st.pool, st.n_slots = object(), S
    monkeypatch.setattr(lsnf4, "layer_pool_prefetch", pool.prefetch)
    monkeypatch.setattr(lsnf4, "layer_pool_acquire", pool.acquire)
    monkeypatch.setattr(lsnf4, "layer_pool_release", pool.release)
    monkeypatch.setattr(lsnf4, "_lib", FakeLib())
    return st, pool


@pytest.mark.parametrize("ahead,api", [(True, "layer"), (False, "layer"), (False, "proj")])
@pytest.mark.parametrize("L,S", [(1, 1), (2, 2), (5, 1), (5, 2), (5, 3), (8, 5), (6, 6), (4, 7), (32, 20), (32, 2)])
def test_sweeps_copy_2L_minus_2S_layers(monkeypatch, L, S, ahead, api):
    st, pool = _cpu_stack(monkeypatch, L, S, ahead, api)
    assert st.ahead == ahead
    counts = []
    for _ in range(3):
        c0, a0 = pool.copies, len(pool.acquired)
        st.step()
        counts.append(pool.copies - c0)
        order = pool.acquired[a0:]
        assert order == list(range(L)) + list(reversed(range(L)))
        assert all(not v for v in pool.held.values()) and sum(pool.refs) == 0
    if S >= L:
        assert counts == [L, 0, 0], counts
    elif S == 1:
        assert counts == [2 * L - 1, 2 * L - 2, 2 * L - 2], counts
    else:
        assert counts == [2 * L - S, 2 * L - 2 * S, 2 * L - 2 * S], counts


@pytest.mark.parametrize("ahead", [True, False])
@pytest.mark.parametrize("L,S", [(6, 2), (6, 4), (32, 20), (32, 2)])
def test_reference_and_recompute_steps_keep_the_pool_consistent(monkeypatch, L, S, ahead):
    """A step with the adapter-off reference forward and the recomputing backward: the reference and the
    policy forward of a layer share one acquisition, so the sweeps acquire each layer once per direction
    and copy as many layers as a plain step (2L - S, then 2L - 2S); no sweep runs out of slots and every
    acquire is released."""
    st, pool = _cpu_stack(monkeypatch, L, S, ahead)
    counts = []
    for _ in range(3):
        a0, c0 = len(pool.acquired), pool.copies
        st.step(reference=True, recompute=True)
        counts.append(pool.copies - c0)
        assert pool.acquired[a0:] == list(range(L)) + list(reversed(range(L)))
        assert sum(pool.refs) == 0
    assert counts == [2 * L - S, 2 * L - 2 * S, 2 * L - 2 * S], counts


def test_layer_layout_splits_codes_and_constants():
    """With resident constants a layer blob is the packed codes alone (4 bits per weight, 1 KiB aligned);
    codes plus constants add up to the whole-blob layout, piece by piece."""
    for name, cfg in synth.STACKS.items():
        codes, lb, cb = layer_layout(cfg, True)
        whole, wb, wcb = layer_layout(cfg, False)
        assert lb + cb == wb and wcb == 0
        for p, q in zip(codes, whole):
            assert p.nbytes + p.cbytes == q.nbytes
            assert p.offset % 1024 == 0 and p.coffset % 1024 == 0
            if cfg.base == "nf4":
                assert p.nbytes == -(-p.N * p.K // 2 // 1024) * 1024
                assert p.cbytes == lsnf4.nf4_blob_bytes(p.N, p.K) - lsnf4.nf4_blob_layout(p.N, p.K)[1]
            else:
                assert p.cbytes == 0 and p.nbytes == -(-p.N * p.K * 2 // 1024) * 1024
    _, lb, cb = layer_layout(synth.STACKS["8b"], True)
    assert (lb, cb) == (109051904, 3468288)          # 8B layer: 109.05 MB streamed, 3.47 MB resident
