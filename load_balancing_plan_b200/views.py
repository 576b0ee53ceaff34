"""Zero-copy views of the receive buffer and their lifetime.

The application works on views of the communication buffer, which the next
dispatch or combine overwrites; a caller that keeps the rows longer (autograd
saving them for the backward pass, for one) must ask for zero_copy = false,
i.e. a copy of its own (twodots.gr "MoonEP balances AI experts in MoE models":
the paragraph on zero-copy communication and static shapes, and the one on
the lifetime of zero-copy views).

RecvView records the workspace's view generation (moonep_view_generation:
dispatch and combine calls launched with that workspace) when it is taken;
reading it after a later dispatch or combine raises StaleViewError instead of
returning rows that belong to another step.  RecvView.copy() is the
zero_copy = false path: moonep_copy_out into a buffer of the caller's.
"""
from . import moonep as mp


class StaleViewError(RuntimeError):
    pass


class RecvView:
    """View of the receive buffer recv ([R * C_max, H] or [R, C_max, H]
    bf16/int16 tensor) written by moonep_dispatch with workspace ws; `rank`
    selects one rank's [C_max, H] rows (None = all ranks)."""

    def __init__(self, cfg, ws, recv, rank=None):
        self.cfg = dict(cfg)
        self.ws = ws
        self._recv = recv
        self.rank = rank
        self.generation = mp.moonep_view_generation(ws)

    def valid(self) -> bool:
        return mp.moonep_view_generation(self.ws) == self.generation

    def _check(self):
        now = mp.moonep_view_generation(self.ws)
        if now != self.generation:
            raise StaleViewError("receive-buffer view taken at generation %d, workspace is at %d: a later "
                                 "dispatch or combine overwrote it (copy it with zero_copy=False first)"
                                 % (self.generation, now))

    @property
    def tensor(self):
        self._check()
        c = self.cfg
        t = self._recv.view(c["R"], c["C_max"], c["H"])
        return t if self.rank is None else t[self.rank]

    def copy(self, out=None, stream=None):
        """zero_copy = false: the rows the plan uses, copied by moonep_copy_out
        into `out` (a new tensor like recv if None; rows the plan does not use
        are left as they were).  Returns a tensor shaped like this view."""
        self._check()
        if out is None:
            import torch
            out = torch.empty_like(self._recv)
        mp.moonep_copy_out(self.cfg, self.ws, self._recv, out, stream)
        c = self.cfg
        t = out.view(c["R"], c["C_max"], c["H"])
        return t if self.rank is None else t[self.rank]
