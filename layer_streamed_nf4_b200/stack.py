"""The layer loop of a training step over a stack of frozen-base LoRA linears.

"Can You Fine-Tune a 27B Model on a Laptop? (I Did the Math)", 7:11-7:42: the
frozen base lives in system RAM, each decoder layer is copied into a small
VRAM buffer on a separate stream while the previous one computes, and every
layer is read twice per step (forward, then backward).  This module drives
that loop through the C ABI: per step a forward sweep over layers 0..L-1
(acquire i, prefetch i+1, seven lora_linear_fwd calls, release i) and a
backward sweep over L-1..0 (acquire i, prefetch i-1, seven lora_linear_bwd
calls, release i).  All compute and all copies are library calls; this file
only sequences them and owns the (synthetic) tensors.

With S pool slots (n_slots) a sweep keeps S layers in flight instead of one:
it prefetches its first S layers at its start and the layer S positions
ahead whenever one is released.  At each turn of the step the S layers the
last sweep used are the first S the next one needs, still resident, so a
step copies 2L-2S layers (2L-4 with the pages' two slots).  S sets how much
of the copy time hides behind compute: on B200 at 2048 tokens a layer's
codes take about twice as long to cross PCIe as its compute.

Two ways to drive a layer (api=...):
  "layer"  one lora_layer_fwd / lora_layer_bwd call per layer and sweep: the
           library launches the seven projections together (one dequant, one
           down-projection and one token-reduction kernel for all of them) and
           the forward keeps u = x A^T for the backward;
  "proj"   seven lora_linear_fwd / lora_linear_bwd calls per layer and sweep.
Both give the same bits.

Dequantisation ahead (dequant_ahead, on by default for NF4 bases with the
layer calls): the weights do not depend on the activations, so while layer i
computes, a side stream acquires layer i+1's slot, runs nf4_dequant on its
projections into one of two bf16 buffers and releases the slot; layer i+1's
call then takes bf16 bases pointing at that buffer.  The dequantisation runs
underneath the previous layer's GEMMs, and a pool slot is held only until
its layer is dequantised.  Same bits as dequantising inside the call.
The dequantisation's grid is capped at ahead_blocks_per_sm blocks per SM
(default 8; a grid-stride loop covers the rest), so that it runs beside the
GEMMs without taking every free slot.  Measured on one B200 (8B shapes, two
slots, whole blobs streamed): with streamed layers the slot returns to the
pool a layer earlier and the copy engine stays busy (122.8 vs 125.6 ms per
step at T = 2048; 212 vs 226 ms at T = 8192); with every layer resident 58.6
vs 58.9 ms.  With the merged GEMM launches, 8 or 16 blocks per SM measured
1-2 ms per step faster than 2 (8B, T = 2048; 1, 4 and an uncapped grid
slower or no better).

Inputs: by default every (layer, projection) has its own x.  With
shared_inputs, q, k and v read one x and gate and up read one x, as in a
decoder layer; with grouped (which implies shared_inputs) those projections
are passed to the layer calls as groups, so each group's forward is one GEMM
over its stacked weights and its backward one GEMM producing the group's
summed input gradient (written to the first member's dX).

Lanes ("proj" only): the seven projections of a layer are independent calls, so they are
issued round-robin on `lanes` streams (default 2), each with its own
workspace.  The side kernels and the dequantisation of one projection then
run underneath another projection's GEMM on the SMs' spare shared memory
and issue slots.  The lanes fork from the compute stream after the layer's
acquire and join it before the layer's release, so the pool's ordering
(release event on the compute stream) is unchanged.  Each call's arithmetic
is independent of the lane it runs on, so results are bitwise the same for
any lane count.

Resident constants (resident_constants, on by default for NF4 bases): a
layer's blob in host RAM holds only the packed codes of its projections;
their double-quantised constants (absmax_q, s2, offset: about 1/32 of the
codes' bytes) stay in device memory for the whole run, so every copy moves codes
only.  The kernels see the same arrays either way (an NF4 weight is four
pointers), so the results are the same bits.

Modes with identical kernels and launch shapes, for the bit-exactness gate
("Exact Layer Streaming", abstract: streamed compared with a resident run of
the same numerics):
  resident  every layer blob copied once into one device buffer;
  streamed  layer blobs in pinned host RAM, n_slots VRAM slots (default 2);
  no_h2d    a pool with one slot per layer, pre-filled before timing.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import lsnf4, synth


def _round_up(a: int, b: int) -> int:
    return (a + b - 1) // b * b


def grad_layout(projs, layers: int, r: int):
    """Element offsets of (dA, dB) of every (layer, projection) in one flat fp32 buffer, and its size:
    per (layer, projection) dA [r, K] then dB [N, r], each starting on a 16-byte boundary."""
    off, n = {}, 0
    for l in range(layers):
        for pi, p in enumerate(projs):
            off[l, pi] = n
            n += r * (p.K + p.N)
            n = _round_up(n, 4)
    return off, n


@dataclass
class ProjLayout:
    name: str
    K: int
    N: int
    offset: int      # byte offset of this projection's streamed bytes in the layer blob
    nbytes: int
    coffset: int = 0  # NF4 with resident constants: byte offset of its constants in the layer's constant block
    cbytes: int = 0


def layer_layout(cfg: synth.StackConfig, resident_constants: bool = True):
    """(projection layouts, streamed bytes per layer, resident constant bytes per layer).  NF4: per
    projection the blob of lsn_nf4_blob_layout, split after the packed codes when the constants stay
    resident; bf16: the row-major matrix.  Every piece starts on a 1 KiB boundary."""
    nf4 = cfg.base == "nf4"
    off = coff = 0
    projs: list[ProjLayout] = []
    for name, K, N in cfg.projections:
        nb, cb = (lsnf4.nf4_blob_bytes(N, K) if nf4 else _round_up(N * K * 2, 1024)), 0
        if nf4 and resident_constants:              # stream the packed codes, keep the constants on the device
            cb = nb - lsnf4.nf4_blob_layout(N, K)[1]
            nb -= cb
        projs.append(ProjLayout(name, K, N, off, nb, coff, cb))
        off += nb
        coff += cb
    return projs, off, coff


class Stack:
    def __init__(self, cfg: synth.StackConfig, layers: int | None = None, tokens: int | None = None,
                 mode: str = "streamed", n_slots: int = 2, seed: int = synth.SEED, keep_outputs: bool = False,
                 distinct_activations: bool = True, device: int = 0, stream: torch.cuda.Stream | None = None,
                 lanes: int = 2, api: str = "layer", shared_inputs: bool = False, grouped: bool = False,
                 dequant_ahead: bool = True, resident_constants: bool = True, ahead_blocks_per_sm: int = 8):
        assert mode in ("resident", "streamed", "no_h2d")
        assert api in ("layer", "proj")
        assert not grouped or api == "layer", "groups are a feature of the layer calls"
        self.api = api
        self.grouped = grouped
        self.shared_inputs = shared_inputs or grouped
        self.cfg, self.mode, self.seed = cfg, mode, seed
        self.L = layers if layers is not None else cfg.layers
        self.T = tokens if tokens is not None else cfg.tokens
        self.r, self.scale = cfg.rank, cfg.alpha / cfg.rank
        self.nf4 = cfg.base == "nf4"
        self.kind = lsnf4.LSN_BASE_NF4 if self.nf4 else lsnf4.LSN_BASE_BF16
        self.dev = torch.device("cuda", device)
        self.stream = stream if stream is not None else torch.cuda.current_stream(self.dev)
        self.keep_outputs = keep_outputs
        assert lanes >= 1
        lanes = lanes if api == "proj" else 1
        self.n_lanes = lanes
        self.lanes = [self.stream] + [torch.cuda.Stream(self.dev) for _ in range(lanes - 1)]
        self._fork = [torch.cuda.Event() for _ in range(lanes)]
        self._join = [torch.cuda.Event() for _ in range(lanes)]
        self.proj, self.layer_bytes, self.const_bytes = layer_layout(cfg, resident_constants)
        self.consts = None
        self.pool = None
        self.host = None
        self.resident = None
        self._calls = {}
        self._distinct = distinct_activations
        self._ahead_opt = dequant_ahead
        assert ahead_blocks_per_sm > 0
        self.ahead_blocks_per_sm = ahead_blocks_per_sm
        self.ahead = self._ahead_for(mode)
        if self.nf4 and api == "layer":
            tot = sum(p.N * p.K for p in self.proj)
            self._wbuf = [torch.empty(tot, dtype=torch.bfloat16, device=self.dev) for _ in range(2)]
            self._woff, o = [], 0
            for p in self.proj:
                self._woff.append(o)
                o += p.N * p.K
            self._prep = torch.cuda.Stream(self.dev)
            self._ev_ready = [torch.cuda.Event() for _ in range(2)]
            self._ev_done = [torch.cuda.Event() for _ in range(2)]
        self._build_weights()
        self._build_tensors(distinct_activations)
        self._setup_mode(n_slots)

    # ------------------------------------------------------------ set-up --

    def _build_weights(self):
        """W ~ N(0, 0.02) per projection, quantised on the device, stored per layer in pinned host RAM
        (with resident constants: the packed codes there, absmax_q / s2 / offset in device memory)."""
        self.host = torch.empty((self.L, self.layer_bytes), dtype=torch.uint8, pin_memory=True)
        dblob = torch.zeros(self.layer_bytes, dtype=torch.uint8, device=self.dev)
        if self.const_bytes:
            self.consts = torch.zeros((self.L, self.const_bytes), dtype=torch.uint8, device=self.dev)
            full = torch.zeros(max(p.nbytes + p.cbytes for p in self.proj), dtype=torch.uint8, device=self.dev)
        maxnk = max(p.N * p.K for p in self.proj)
        qws_bytes = lsnf4.nf4_quantize_ws_bytes(1, maxnk) if self.nf4 else 0
        qws = torch.zeros(max(qws_bytes, 16), dtype=torch.uint8, device=self.dev)
        with torch.cuda.stream(self.stream):
            for l in range(self.L):
                for pi, p in enumerate(self.proj):
                    W = synth.device_normal((p.N, p.K), 0.02, self.seed, l, pi, synth.T_W, device=self.dev)
                    if self.nf4 and p.cbytes:           # quantise into one full blob, then split it
                        w = lsnf4.nf4_weight_in_blob(p.N, p.K, full.data_ptr())
                        lsnf4.nf4_quantize(W, w, qws, qws_bytes, self.stream)
                        dblob[p.offset:p.offset + p.nbytes].copy_(full[:p.nbytes])
                        self.consts[l, p.coffset:p.coffset + p.cbytes].copy_(full[p.nbytes:p.nbytes + p.cbytes])
                    elif self.nf4:
                        w = lsnf4.nf4_weight_in_blob(p.N, p.K, dblob.data_ptr() + p.offset)
                        lsnf4.nf4_quantize(W, w, qws, qws_bytes, self.stream)
                    else:
                        dst = dblob[p.offset:p.offset + p.N * p.K * 2].view(torch.bfloat16)
                        dst.copy_(W.reshape(-1).to(torch.bfloat16))
                    del W
                self.host[l].copy_(dblob, non_blocking=False)
        self.stream.synchronize()

    def _build_tensors(self, distinct: bool):
        T, r, dev = self.T, self.r, self.dev
        self.x, self.dY, self.A, self.B, self.dA, self.dB = {}, {}, {}, {}, {}, {}
        # every dA [r, K] and dB [N, r] of the stack in one fp32 buffer, so that data-parallel
        # replicas sum them with one collective
        self.grad_offsets, n = grad_layout(self.proj, self.L, r)
        self.grads = torch.zeros(n, dtype=torch.float32, device=dev)
        h0 = None
        if self.cfg.vocab:
            # Layer 0 reads token embeddings: rows of a resident N(0, 1) bf16 table [vocab, hidden] picked by T
            # token ids uniform over the vocabulary.  q, k and v take them as their input (the layer's input
            # norm is not part of the linears).
            self.token_ids = synth.device_token_ids(T, self.cfg.vocab, self.seed, device=dev)
            self.embedding = synth.device_normal((self.cfg.vocab, self.cfg.hidden), 1.0, self.seed, synth.T_EMB,
                                                 device=dev, dtype=torch.bfloat16)
            h0 = self.embedding.index_select(0, self.token_ids)
        for l in range(self.L):
            for pi, p in enumerate(self.proj):
                la = l if distinct else 0
                src = self._input_of(pi)
                if src != pi:                                   # shares the x of an earlier projection
                    self.x[l, pi] = self.x[l, src]
                elif l == 0 and h0 is not None and p.name in ("q", "k", "v"):
                    self.x[l, pi] = h0
                else:
                    self.x[l, pi] = synth.device_normal((T, p.K), 1.0, self.seed, la, pi, synth.T_X, device=dev,
                                                        dtype=torch.bfloat16) if (distinct or l == 0) else self.x[0, pi]
                self.dY[l, pi] = synth.device_normal((T, p.N), 1.0, self.seed, la, pi, synth.T_DY, device=dev,
                                                     dtype=torch.bfloat16) if (distinct or l == 0) else self.dY[0, pi]
                self.A[l, pi] = synth.device_uniform((r, p.K), 1.0 / p.K ** 0.5, self.seed, l, pi, synth.T_A,
                                                     device=dev, dtype=torch.bfloat16)
                self.B[l, pi] = synth.device_normal((p.N, r), 0.01, self.seed, l, pi, synth.T_B, device=dev,
                                                    dtype=torch.bfloat16)
                o = self.grad_offsets[l, pi]
                self.dA[l, pi] = self.grads[o:o + r * p.K].view(r, p.K)
                self.dB[l, pi] = self.grads[o + r * p.K:o + r * (p.K + p.N)].view(p.N, r)
        nl = self.L if self.keep_outputs else 1
        self.y = {(l, pi): torch.empty((T, p.N), dtype=torch.bfloat16, device=dev)
                  for l in range(nl) for pi, p in enumerate(self.proj)}
        self.dX = {(l, pi): torch.empty((T, p.K), dtype=torch.bfloat16, device=dev)
                   for l in range(nl) for pi, p in enumerate(self.proj)}
        self.y_ref = {(l, pi): torch.empty((T, p.N), dtype=torch.bfloat16, device=dev)
                      for l in range(nl) for pi, p in enumerate(self.proj)}
        if self.api == "layer":
            # u = x A^T kept from the forward for the backward, per (layer, projection)
            self.u = {(l, pi): torch.zeros((T, r), dtype=torch.float32, device=dev)
                      for l in range(self.L) for pi in range(len(self.proj))}
            self.ws_bytes = lsnf4.layer_ws_bytes(self._layer_projs(0, 0), T, r)
        else:
            self.ws_bytes = max(lsnf4.lora_ws_bytes(T, p.K, p.N, r, self.kind) for p in self.proj)
        self.ws = [torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev) for _ in range(self.n_lanes)]
        torch.cuda.synchronize(dev)

    def _setup_mode(self, n_slots: int):
        if self.mode == "resident":
            self.resident = self.host.to(self.dev)
            self.n_slots = self.L
            return
        slots = self.L if self.mode == "no_h2d" else n_slots
        self.n_slots = slots
        self.pool = lsnf4.layer_pool_create(slots, self.layer_bytes, self.dev.index or 0)
        for l in range(self.L):
            lsnf4.layer_pool_register(self.pool, l, self.host[l].data_ptr(), self.layer_bytes)
        if self.mode == "no_h2d":
            for l in range(self.L):
                lsnf4.layer_pool_prefetch(self.pool, l)
            lsnf4.layer_pool_wait_idle(self.pool, 600000)

    def with_mode(self, mode: str, n_slots: int = 2, lanes: int | None = None, api: str | None = None) -> "Stack":
        """A stack sharing this one's host blobs and tensors, run in another mode
        (and, if given, another lane count)."""
        import copy
        assert mode in ("resident", "streamed", "no_h2d")
        other = copy.copy(self)
        other.mode, other.pool, other.resident, other._calls = mode, None, None, {}
        other.ahead = other._ahead_for(mode)
        if api is not None and api != self.api:
            assert api == "proj" or hasattr(self, "u"), "a stack built for the per-projection calls keeps no u"
            other.api = api
            if api == "layer":
                other.ws_bytes = lsnf4.layer_ws_bytes(self._layer_projs(0, 0), self.T, self.r)
            else:
                other.ws_bytes = max(lsnf4.lora_ws_bytes(self.T, p.K, p.N, self.r, self.kind) for p in self.proj)
            other.n_lanes = lanes if (lanes is not None and api == "proj") else 1
            other.lanes = [self.stream] + [torch.cuda.Stream(self.dev) for _ in range(other.n_lanes - 1)]
            other._fork = [torch.cuda.Event() for _ in range(other.n_lanes)]
            other._join = [torch.cuda.Event() for _ in range(other.n_lanes)]
            other.ws = [torch.zeros(other.ws_bytes, dtype=torch.uint8, device=self.dev) for _ in range(other.n_lanes)]
        elif lanes is not None and lanes != self.n_lanes and self.api == "proj":
            other.n_lanes = lanes
            other.lanes = [self.stream] + [torch.cuda.Stream(self.dev) for _ in range(lanes - 1)]
            other._fork = [torch.cuda.Event() for _ in range(lanes)]
            other._join = [torch.cuda.Event() for _ in range(lanes)]
            other.ws = [torch.zeros(self.ws_bytes, dtype=torch.uint8, device=self.dev) for _ in range(lanes)]
        other._setup_mode(n_slots)
        return other

    def with_tokens(self, tokens: int, mode: str = "streamed", n_slots: int = 2) -> "Stack":
        """A stack sharing this one's host blobs (the frozen base) and adapters' seeds, with its own
        activations for `tokens` tokens (a larger batch streams the same weights)."""
        import copy
        other = copy.copy(self)
        other.T, other.mode = tokens, mode
        other.pool, other.resident, other._calls = None, None, {}
        other.ahead = other._ahead_for(mode)
        other._build_tensors(self._distinct)
        other._setup_mode(n_slots)
        return other

    def close(self):
        if self.pool is not None:
            lsnf4.layer_pool_destroy(self.pool)
            self.pool = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ layers --

    def _acquire(self, l: int, stream=None) -> int:
        if self.mode == "resident":
            return self.resident[l].data_ptr()
        return lsnf4.layer_pool_acquire(self.pool, l, stream or self.stream)

    def _prefetch(self, l: int):
        if self.mode != "resident" and 0 <= l < self.L:
            lsnf4.layer_pool_prefetch(self.pool, l)

    def _window(self, order):
        """fill(pos): prefetch the layers at positions <= pos of a sweep, each once.  A sweep keeps
        the pool's S slots busy: its first S layers at the start (at a turn these are the S layers the
        previous sweep used last, still resident), then one more whenever a layer has been released."""
        nxt = 0

        def fill(pos):
            nonlocal nxt
            while nxt < len(order) and nxt <= pos:
                self._prefetch(order[nxt])
                nxt += 1
        return fill

    def _release(self, l: int, stream=None):
        if self.mode != "resident":
            lsnf4.layer_pool_release(self.pool, l, stream or self.stream)

    def _nf4_view(self, addr: int, l: int, p: ProjLayout) -> lsnf4.NF4Weight:
        """Projection p of layer l, its blob bytes at addr (and its constants in the resident block)."""
        if not p.cbytes:
            return lsnf4.nf4_weight_in_blob(p.N, p.K, addr + p.offset)
        o = lsnf4.nf4_blob_layout(p.N, p.K)
        c = self.consts[l].data_ptr() + p.coffset - o[1]
        return lsnf4.NF4Weight(p.N, p.K, addr + p.offset, c + o[1], c + o[2], c + o[3])

    def _base(self, addr: int, l: int, p: ProjLayout):
        if self.nf4:
            return lsnf4.base_nf4(self._nf4_view(addr, l, p))
        return lsnf4.base_bf16(addr + p.offset, p.N, p.K)

    def _out(self, d, l, pi):
        return d[(l if self.keep_outputs else 0), pi]

    def _fork_lanes(self):
        """Lanes 1.. start after what the compute stream has issued (the acquire)."""
        if self.n_lanes > 1:
            self._fork[0].record(self.stream)
            for ln in self.lanes[1:]:
                ln.wait_event(self._fork[0])

    def _join_lanes(self):
        """The compute stream continues after every lane's work on the layer."""
        for i, ln in enumerate(self.lanes[1:], 1):
            self._join[i].record(ln)
            self.stream.wait_event(self._join[i])

    # The per-call arguments depend only on (slot address, layer, projection),
    # so they are marshalled once and the C entry points are called directly.

    def _fwd_args(self, addr: int, l: int, pi: int):
        key = ("f", addr, l, pi)
        a = self._calls.get(key)
        if a is None:
            p = self.proj[pi]
            base = self._base(addr, l, p)
            lane = pi % self.n_lanes
            a = (ctypes.byref(base), self.x[l, pi].data_ptr(), self.T, self.A[l, pi].data_ptr(),
                 self.B[l, pi].data_ptr(), self.r, self.scale, self._out(self.y, l, pi).data_ptr(),
                 self.ws[lane].data_ptr(), self.ws_bytes, self.lanes[lane].cuda_stream, base)
            self._calls[key] = a
        return a

    def _bwd_args(self, addr: int, l: int, pi: int, accumulate: bool):
        key = ("b", addr, l, pi, accumulate)
        a = self._calls.get(key)
        if a is None:
            p = self.proj[pi]
            base = self._base(addr, l, p)
            lane = (len(self.proj) - 1 - pi) % self.n_lanes
            a = (ctypes.byref(base), self.x[l, pi].data_ptr(), self.dY[l, pi].data_ptr(), self.T,
                 self.A[l, pi].data_ptr(), self.B[l, pi].data_ptr(), self.r, self.scale,
                 self._out(self.dX, l, pi).data_ptr(), self.dA[l, pi].data_ptr(), self.dB[l, pi].data_ptr(),
                 int(accumulate), self.ws[lane].data_ptr(), self.ws_bytes, self.lanes[lane].cuda_stream, base)
            self._calls[key] = a
        return a

    # q, k, v read the input of q; gate and up the input of gate (index into the projection list)
    _GROUP_OF = {"q": 1, "k": 1, "v": 1, "gate": 2, "up": 2}
    _INPUT_OF = {"k": "q", "v": "q", "up": "gate"}

    def _input_of(self, pi: int) -> int:
        if not self.shared_inputs:
            return pi
        names = [p.name for p in self.proj]
        src = self._INPUT_OF.get(names[pi])
        return names.index(src) if src in names else pi

    def _group_of(self, pi: int) -> int:
        return self._GROUP_OF.get(self.proj[pi].name, 0) if self.grouped else 0

    def _leads(self, pi: int) -> bool:
        g = self._group_of(pi)
        return g == 0 or pi == 0 or self._group_of(pi - 1) != g

    def with_inputs(self, shared_inputs: bool = True, grouped: bool = False, mode: str = "no_h2d",
                    n_slots: int = 2) -> "Stack":
        """A stack sharing this one's host blobs, with its own activations: shared inputs per group of
        projections, and (grouped) the groups passed to the layer calls."""
        import copy
        other = copy.copy(self)
        other.shared_inputs, other.grouped = shared_inputs or grouped, grouped
        other.mode, other.pool, other.resident, other._calls = mode, None, None, {}
        other.ahead = other._ahead_for(mode)
        other._build_tensors(self._distinct)
        other._setup_mode(n_slots)
        return other

    def ahead_on_compute_stream(self):
        """Run the dequantisation ahead on the compute stream, serialised with the layer calls, instead of on
        its side stream: the same launches on one lane (for per-launch timing)."""
        if self.ahead:
            self._prep = self.stream

    def _ahead_for(self, mode: str) -> bool:
        return bool(self._ahead_opt and self.nf4 and self.api == "layer")

    def _ahead_base(self, b: int, pi: int):
        p = self.proj[pi]
        return lsnf4.base_bf16(self._wbuf[b].data_ptr() + 2 * self._woff[pi], p.N, p.K)

    def _layer_projs(self, addr: int, l: int, adapter: bool = True, wb: int | None = None):
        """The lsn_lora_proj array of layer l whose blob sits at addr (cached: it depends on nothing else).
        adapter=False: A and B NULL, the frozen base alone (the reference model of preference training).
        wb: bf16 bases in dequantisation buffer wb instead of the NF4 blob."""
        key = ("L", addr, l, adapter, wb)
        a = self._calls.get(key)
        if a is None:
            projs = [lsnf4.lora_proj(self._base(addr, l, p) if wb is None else self._ahead_base(wb, pi), self.x[l, pi],
                                     self.A[l, pi] if adapter else None, self.B[l, pi] if adapter else None,
                                     y=self._out(self.y if adapter else self.y_ref, l, pi), dY=self.dY[l, pi],
                                     dX=self._out(self.dX, l, pi) if self._leads(pi) else None,
                                     dA=self.dA[l, pi], dB=self.dB[l, pi],
                                     u=self.u[l, pi] if (adapter and hasattr(self, "u")) else None,
                                     group=self._group_of(pi))
                     for pi, p in enumerate(self.proj)]
            a = lsnf4.proj_array(projs)
            if addr or wb is not None:
                self._calls[key] = a
        return a

    def _prep_layer(self, l: int, b: int):
        """On the side stream: wait until buffer b is free, acquire layer l's slot, dequantise its
        projections into buffer b, release the slot, mark buffer b ready."""
        ps = self._prep
        ps.wait_event(self._ev_done[b])
        addr = self._acquire(l, ps)
        key = ("D", addr, l, b)
        args = self._calls.get(key)
        if args is None:                          # one launch for the layer's projections
            ws = [self._nf4_view(addr, l, p) for p in self.proj]
            outs = [self._wbuf[b].data_ptr() + 2 * self._woff[pi] for pi in range(len(self.proj))]
            args = self._calls[key] = lsnf4.dequant_batch_args(ws, outs)
        # a capped grid: the dequantisation runs beside the current layer's GEMMs
        st = lsnf4._lib.nf4_dequant_batch(*args, self.ahead_blocks_per_sm, ps.cuda_stream)
        if st:
            lsnf4._check(st, "nf4_dequant_batch")
        self._release(l, ps)
        self._ev_ready[b].record(ps)

    def _sweep_ahead(self, order, call):
        """Run call(l, projs) over the layers in `order`, each layer dequantised one layer ahead.
        The slot of position j is released once j is dequantised, so position j + S may be prefetched."""
        order = list(order)
        if not order:
            return
        S = self.n_slots
        fill = self._window(order)
        fill(S - 1)
        self._prep_layer(order[0], 0)
        fill(S)
        for idx, l in enumerate(order):
            b = idx % 2
            if idx + 1 < len(order):
                self._prep_layer(order[idx + 1], (idx + 1) % 2)
                fill(idx + 1 + S)
            self.stream.wait_event(self._ev_ready[b])
            call(l, b)
            self._ev_done[b].record(self.stream)

    def _forward_layers(self, adapter: bool = True, reference: bool = False):
        """Forward sweep through the layer calls.  reference: each layer runs twice while it is held, first
        with the adapters off (the reference model's forward, into y_ref), then with them on: two
        independent forward passes sharing one read of the layer stream."""
        fwd = lsnf4._lib.lora_layer_fwd
        n, ws, nb, sp = len(self.proj), self.ws[0].data_ptr(), self.ws_bytes, self.stream.cuda_stream
        passes = (False, True) if reference else (adapter,)
        # With the forward GEMMs converting NF4 in tensor memory (LSN_OPT_FUSED_NF4 = 2) the forward sweep
        # hands the layer calls the NF4 codes themselves; only the backward sweep dequantises ahead.
        if self.ahead and lsnf4.get_option(lsnf4.LSN_OPT_FUSED_NF4) != 2:
            def call(l, b):
                for ad in passes:
                    st = fwd(n, self._layer_projs(0, l, ad, wb=b), self.T, self.r, self.scale, ws, nb, sp)
                    if st:
                        lsnf4._check(st, "lora_layer_fwd")
            return self._sweep_ahead(range(self.L), call)
        order = list(range(self.L))
        fill = self._window(order)
        fill(self.n_slots - 1)
        for j, l in enumerate(order):
            addr = self._acquire(l)
            fill(j + self.n_slots - 1)
            for ad in passes:
                st = fwd(n, self._layer_projs(addr, l, ad), self.T, self.r, self.scale, ws, nb, sp)
                if st:
                    lsnf4._check(st, "lora_layer_fwd")
            self._release(l)

    def _backward_layers(self, accumulate: bool, recompute: bool = False):
        fwd, bwd = lsnf4._lib.lora_layer_fwd, lsnf4._lib.lora_layer_bwd
        n, ws, nb, sp = len(self.proj), self.ws[0].data_ptr(), self.ws_bytes, self.stream.cuda_stream
        if self.ahead:
            def call(l, b):
                projs = self._layer_projs(0, l, wb=b)
                if recompute:
                    st = fwd(n, projs, self.T, self.r, self.scale, ws, nb, sp)
                    if st:
                        lsnf4._check(st, "lora_layer_fwd")
                st = bwd(n, projs, self.T, self.r, self.scale, int(accumulate), ws, nb, sp)
                if st:
                    lsnf4._check(st, "lora_layer_bwd")
            return self._sweep_ahead(reversed(range(self.L)), call)
        order = list(reversed(range(self.L)))
        fill = self._window(order)
        fill(self.n_slots - 1)
        for j, l in enumerate(order):
            addr = self._acquire(l)
            fill(j + self.n_slots - 1)
            projs = self._layer_projs(addr, l)
            if recompute:     # the layer's forward again, inside the backward sweep (activation checkpointing)
                st = fwd(n, projs, self.T, self.r, self.scale, ws, nb, sp)
                if st:
                    lsnf4._check(st, "lora_layer_fwd")
            st = bwd(n, projs, self.T, self.r, self.scale, int(accumulate), ws, nb, sp)
            if st:
                lsnf4._check(st, "lora_layer_bwd")
            self._release(l)

    def forward(self, adapter: bool = True, reference: bool = False):
        if self.api == "layer":
            return self._forward_layers(adapter, reference)
        assert adapter and not reference, "the adapter-off forward runs through the layer calls"
        fwd = lsnf4._lib.lora_linear_fwd
        order = list(range(self.L))
        fill = self._window(order)
        fill(self.n_slots - 1)
        for j, l in enumerate(order):
            addr = self._acquire(l)
            fill(j + self.n_slots - 1)
            self._fork_lanes()
            for pi in range(len(self.proj)):
                st = fwd(*self._fwd_args(addr, l, pi)[:-1])
                if st:
                    lsnf4._check(st, "lora_linear_fwd")
            self._join_lanes()
            self._release(l)

    def backward(self, accumulate: bool = False, recompute: bool = False):
        if self.api == "layer":
            return self._backward_layers(accumulate, recompute)
        assert not recompute, "the recomputing backward runs through the layer calls"
        bwd = lsnf4._lib.lora_linear_bwd
        order = list(reversed(range(self.L)))
        fill = self._window(order)
        fill(self.n_slots - 1)
        for j, l in enumerate(order):
            addr = self._acquire(l)
            fill(j + self.n_slots - 1)
            self._fork_lanes()
            for pi in reversed(range(len(self.proj))):
                st = bwd(*self._bwd_args(addr, l, pi, accumulate)[:-1])
                if st:
                    lsnf4._check(st, "lora_linear_bwd")
            self._join_lanes()
            self._release(l)

    def step(self, accumulate: bool = False, reference: bool = False, recompute: bool = False):
        """One training step.  reference: the forward sweep also runs every layer with the adapters off (the
        reference model of preference training, on the same stream of layers: each layer is read once for
        both forwards, so the step copies as many layers as a plain one); recompute: every layer's forward
        runs again inside the backward sweep, as with activation checkpointing."""
        self.forward(reference=reference)
        self.backward(accumulate, recompute)

    # ------------------------------------------------------------ facts ---

    def flop_per_step(self) -> float:
        return float(self.cfg.flop_per_token_per_layer()) * self.T * self.L

    def h2d_bytes_per_layer(self) -> int:
        return self.layer_bytes

    def pool_stats(self) -> dict | None:
        return lsnf4.layer_pool_stats(self.pool) if self.pool is not None else None

    def check_status(self):
        for ws, ln in zip(self.ws, self.lanes):
            lsnf4.ws_status(ws, ln)


class HostIO:
    """Steps whose inputs come from pinned host memory and whose result goes back to it.

    Each step reads its layer-0 projection inputs from the stack's device tensors (x[0, p]) and leaves its
    layer-0 input gradients in dX[0, p].  Every step's inputs cross PCIe host-to-device and its result
    device-to-host, on a copy stream of their own and through device staging buffers, so that the
    transfers overlap the neighbouring steps' compute: while step k runs, the copy stream brings step k+1's
    inputs into the input staging buffer and sends step k-1's gradients from the output staging buffer to
    the host.  The compute stream adds only two device-to-device copies per step (staging -> x[0, p] before
    the step, dX[0, p] -> staging after it).  The first step's inputs and the last step's result are
    waited for: `run` returns with every transfer ordered before the compute stream's next work.
    """

    @staticmethod
    def inputs_of(stack: "Stack") -> list:
        """The step's input tensors: x[0, p] of each projection that has its own (q, k, v share one with
        shared inputs)."""
        return [stack.x[0, pi] for pi in range(len(stack.proj)) if stack._input_of(pi) == pi]

    @staticmethod
    def outputs_of(stack: "Stack") -> list:
        """The step's result: dX[0, p] of each projection that writes one (a group's first member)."""
        return [stack.dX[0, pi] for pi in range(len(stack.proj)) if stack._leads(pi)]

    @staticmethod
    def host_buffers(stack: "Stack"):
        """Pinned host buffers for inputs_of (holding the device inputs' current values) and outputs_of."""
        h_in = [torch.empty_like(t, device="cpu").pin_memory() for t in HostIO.inputs_of(stack)]
        for h, t in zip(h_in, HostIO.inputs_of(stack)):
            h.copy_(t)
        h_out = [torch.empty_like(t, device="cpu").pin_memory() for t in HostIO.outputs_of(stack)]
        return h_in, h_out

    def __init__(self, stack: "Stack", h_in, h_out, stream=None):
        """stream: the stream the steps run on (default: the stack's)."""
        self.stack = stack
        self.compute = stream or stack.stream
        self.copy = torch.cuda.Stream(stack.dev)
        self.ins = self.inputs_of(stack)
        self.outs = self.outputs_of(stack)
        if len(h_in) != len(self.ins) or len(h_out) != len(self.outs):
            raise ValueError("HostIO: one host buffer per input tensor and per result tensor expected")
        for h, t in list(zip(h_in, self.ins)) + list(zip(h_out, self.outs)):
            if h.device.type != "cpu" or not h.is_pinned() or h.shape != t.shape or h.dtype != t.dtype:
                raise ValueError("HostIO: host buffers must be pinned CPU tensors of the device tensors' shape and "
                                 "dtype")
        self.h_in, self.h_out = list(h_in), list(h_out)
        self.stage_in = [torch.empty_like(t) for t in self.ins]
        self.stage_out = [torch.empty_like(t) for t in self.outs]
        self.in_ready, self.in_free = torch.cuda.Event(), torch.cuda.Event()
        self.out_ready, self.out_free = torch.cuda.Event(), torch.cuda.Event()

    def bytes_in(self) -> int:
        return sum(h.numel() * h.element_size() for h in self.h_in)

    def bytes_out(self) -> int:
        return sum(h.numel() * h.element_size() for h in self.h_out)

    def _h2d(self):
        with torch.cuda.stream(self.copy):
            for h, s in zip(self.h_in, self.stage_in):
                s.copy_(h, non_blocking=True)
            self.in_ready.record(self.copy)

    def run(self, steps: int, step_fn):
        """`steps` calls of step_fn() on the compute stream, each on inputs copied in from the host and each
        followed by the copy of its result to the host."""
        if steps <= 0:
            return
        c, cp = self.compute, self.copy
        cp.wait_stream(c)                          # the staging buffers are free of earlier work
        self._h2d()
        for k in range(steps):
            c.wait_event(self.in_ready)
            with torch.cuda.stream(c):
                for s, t in zip(self.stage_in, self.ins):
                    t.copy_(s, non_blocking=True)
            self.in_free.record(c)
            if k + 1 < steps:                      # the next step's inputs, beside this step's compute
                cp.wait_event(self.in_free)
                self._h2d()
            with torch.cuda.stream(c):
                step_fn()
                if k > 0:
                    c.wait_event(self.out_free)    # the previous result has left the staging buffer
                for t, s in zip(self.outs, self.stage_out):
                    s.copy_(t, non_blocking=True)
            self.out_ready.record(c)
            cp.wait_event(self.out_ready)
            with torch.cuda.stream(cp):
                for s, h in zip(self.stage_out, self.h_out):
                    h.copy_(s, non_blocking=True)
                self.out_free.record(cp)
        c.wait_event(self.out_free)                # the last result is on the host
