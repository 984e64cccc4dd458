"""Drive the whole device path for one synthetic workload through the C ABI.

prefill (synthetic, dense) -> seed_state_init_from_dense -> per step and layer:
seed_synth_token_inputs + seed_decode_step, and seed_compress after the step that
fills R + W columns (every W steps, decode steps counted from 1).  With ragged
schedules the requests joined at different times (a lead-in of up to W - 1 steps)
and seed_compress runs after every step, compressing the units that are due.  With
fused=True the step after which a compression is due (every step when ragged) is
seed_decode_step_compress, which compresses the due units inside the decode launch.

Every step of the path runs in libseed's kernels; this module only allocates
tensors, orders the calls and tracks the (uniform) column count on the host.
"""

from __future__ import annotations

import torch

from . import seed as S


class DeviceRun:
    """One workload resident on the device: v̄, the stored state and a workspace."""

    def __init__(self, cfg, batch: int | None = None, b0: int = 0, device: str = "cuda",
                 n_prefill: int | None = None, keep_dense: bool = False, ragged: bool = False,
                 factors: int = S.SEED_FACTORS_F32, fused: bool = False, overlap: bool = False):
        self.cfg = cfg
        self.dims = S.Dims.from_config(cfg, batch, factors)
        self.key = S.synth_key(cfg, b0)
        self.device = device
        d = self.dims
        self.ws = S.Workspace(d, device)
        self.vbar = torch.empty(d.layers, d.heads, d.d_v, dtype=torch.float32, device=device)
        S.seed_synth_vbar(d, self.key, self.vbar)
        self.state = S.State.allocate(d, self.vbar)
        self.n_prefill = cfg.n_prefill if n_prefill is None else n_prefill
        self.dense = None
        self.sigma_conv = None
        self.c = 0
        self.t = 0
        self.keep_dense = keep_dense
        # ragged schedules: request b (global index) joined phi_b steps before the
        # others, phi_b = W - 1 - floor(b W / B) for the workload's B requests, so the
        # requests still in their lead-in at lead-in step j are a prefix of the batch
        self.ragged = ragged
        self.fused = fused
        # layers after the first use seed_decode_step_overlapped: the launch before
        # each is the previous layer's step, which writes none of its state (the
        # first layer may follow a compression)
        self.overlap = overlap
        gb = torch.arange(b0, b0 + self.dims.batch)
        self.phase = (cfg.W - 1 - (gb * cfg.W) // cfg.batch).clamp(min=0) if ragged else torch.zeros_like(gb)

    # ------------------------------------------------------------------ setup
    def prefill_and_convert(self, layer_chunk: int | None = None) -> None:
        """Dense prefill of every unit, then the end-of-prefill conversion."""
        d = self.dims
        per_layer = d.batch * d.heads * d.d_k * d.d_v
        if self.keep_dense:
            self.dense = torch.empty(d.batch, d.layers, d.heads, d.d_k, d.d_v, dtype=torch.float32,
                                     device=self.device)
        self.sigma_conv = torch.empty(d.batch, d.layers, d.heads, d.R, dtype=torch.float32,
                                      device=self.device)
        buf = torch.empty(per_layer, dtype=torch.float32, device=self.device)
        sig = torch.empty(d.batch * d.heads * d.R, dtype=torch.float32, device=self.device)
        for l in range(d.layers):
            S.seed_synth_dense_prefill(d, self.key, self.n_prefill, l, self.vbar, buf)
            S.seed_state_init_from_dense(d, self.state, l, buf, self.ws, sigma_out=sig)
            self.sigma_conv[:, l] = sig.view(d.batch, d.heads, d.R)
            if self.keep_dense:
                self.dense[:, l] = buf.view(d.batch, d.heads, d.d_k, d.d_v)
        self.c = d.R
        self.t = 0

    def lead_in(self, buf: dict) -> None:
        """Ragged schedules: request b takes phi_b decode steps (lead-in inputs, t = 0 ..
        phi_b - 1) before step 0, launched over the batch prefix still leading in."""
        d = self.dims
        for j in range(self.cfg.W - 1):
            nb = int((self.phase > j).sum())
            if nb == 0:
                break
            dj = S.Dims(d.form, nb, d.layers, d.heads, d.d_k, d.d_v, d.R, d.W, d.factors)
            bj = {k: (None if x is None else x[:nb]) for k, x in buf.items()}
            for l in range(d.layers):
                S.seed_synth_token_inputs(dj, self.key, S.SEED_PHASE_LEADIN, j, l, self.vbar,
                                          bj["q"], bj["k"], bj["v"], bj["alpha"], bj["beta"])
                S.seed_decode_step(dj, self.state, l, bj["q"], bj["k"], bj["v"], bj["alpha"], bj["beta"],
                                   bj["o"], self.ws)

    # ------------------------------------------------------------------ decode
    def gen_inputs(self, t: int, layer: int, buf: dict) -> None:
        S.seed_synth_token_inputs(self.dims, self.key, S.SEED_PHASE_DECODE, t, layer, self.vbar,
                                  buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"])

    def step(self, buf: dict, outs: list | None = None, sigma: torch.Tensor | None = None,
             dense: bool = False, pre_compress=None) -> bool:
        """One decode step of every layer (inputs generated on the device), then the
        compression if it is due.  Returns True when a compression ran.  pre_compress:
        called with no argument right before a separate compression launch (not with
        the fused step), e.g. to read the states about to be compressed."""
        d = self.dims
        fuse = self.fused and (self.ragged or self.c + 1 == d.m)
        sig_l = None
        if fuse and sigma is not None:
            sig_l = torch.empty(d.batch * d.heads, d.R, dtype=torch.float32, device=self.device)
        for l in range(d.layers):
            self.gen_inputs(self.t, l, buf)
            if fuse:
                if sig_l is not None:   # keep the rows of units this step does not compress
                    sig_l.copy_(sigma.view(d.batch, d.layers, d.heads, d.R)[:, l].reshape(-1, d.R))
                S.seed_decode_step_compress(d, self.state, l, buf["q"], buf["k"], buf["v"], buf["alpha"],
                                            buf["beta"], buf["o"], self.ws, sigma_out=sig_l)
                if sig_l is not None:
                    sigma.view(d.batch, d.layers, d.heads, d.R)[:, l] = sig_l.view(d.batch, d.heads, d.R)
            else:
                step = S.seed_decode_step_overlapped if (self.overlap and l > 0) else S.seed_decode_step
                step(d, self.state, l, buf["q"], buf["k"], buf["v"], buf["alpha"], buf["beta"], buf["o"], self.ws)
            if dense and self.dense is not None:
                S.seed_dense_step(d, self.dense, l, buf["q"], buf["k"], buf["v"], buf["alpha"],
                                  buf["beta"], buf["o_dense"], self.ws)
            if outs is not None:
                outs[l] = buf["o"].clone()
        self.c += 1
        self.t += 1
        if self.ragged:   # some request is due after every step: only its units compress
            if not fuse:
                if pre_compress is not None:
                    pre_compress()
                S.seed_compress(d, self.state, S.SEED_ALL_LAYERS, self.ws, sigma_out=sigma)
            return True
        if self.c == d.m:
            if not fuse:
                if pre_compress is not None:
                    pre_compress()
                S.seed_compress(d, self.state, S.SEED_ALL_LAYERS, self.ws, sigma_out=sigma)
            self.c = d.R
            return True
        return False

    def to_dense(self, units: torch.Tensor | None = None) -> torch.Tensor:
        """Dense states of all units (or the listed global unit indices)."""
        d = self.dims
        n = d.units if units is None else int(units.numel())
        out = torch.empty(n, d.d_k, d.d_v, dtype=torch.float32, device=self.device)
        S.seed_state_to_dense(d, self.state, S.SEED_ALL_LAYERS, out, self.ws, units=units)
        return out

    def status(self) -> int:
        return S.seed_get_status(self.ws)
