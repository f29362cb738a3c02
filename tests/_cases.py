"""Builds one seeded case for both sides: device tensors for the library, float64 arrays of the
very same stored values for the oracle. Storage rounding (fp32 -> bf16, round to nearest even)
happens once, here, through torch; nothing in this file computes attention."""
from __future__ import annotations

import numpy as np
import torch

import synth

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}

# parity bars: max|Δ| / max|ref| of the outputs, and |Δ lse| (fp32: relative to max(1, max|lse|))
TOL = {"f32": dict(out=1e-5, lse=1e-5), "bf16": dict(out=2e-2, lse=1e-3)}


def stored(a: np.ndarray, dtype: str):
    """(torch CPU tensor in storage dtype, float64 numpy view of the stored values)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(TORCH_DT[dtype])
    return t, t.to(torch.float64).numpy()


class Case:
    """Host-side inputs of one decode step; `to_device()` uploads them."""

    def __init__(self, w: synth.Workload, lens=None, with_weights=True):
        self.w = w
        self.lens = synth.seq_lengths(w) if lens is None else np.asarray(lens, np.int32)
        self.table, self.num_pages = synth.block_table(w, self.lens)
        self.row_off = np.concatenate([[0], np.cumsum(self.lens.astype(np.int64))])
        dt = w.dtype
        tdt = TORCH_DT[dt]
        total = int(self.row_off[-1])
        # pool of interleaved rows [latent | rope], filled through the page table
        self.pool = torch.zeros(self.num_pages * 64, w.d_c + w.d_r, dtype=tdt)
        pool_idx = self.pool_rows()
        for start, c, kr in synth.cache_row_chunks(w, total):
            n = len(c)
            rows = torch.from_numpy(np.concatenate([c, kr], axis=1)).to(tdt)
            self.pool[torch.from_numpy(pool_idx[start:start + n])] = rows
        step = synth.decode_step_inputs(w)
        self.x, self.x64 = stored(step["x"], dt)
        self.q_nope, self.q_nope64 = stored(step["q_nope"], dt)
        self.q_rope_raw, self.q_rope_raw64 = stored(step["q_rope_raw"], dt)
        self.q_abs, self.q_abs64 = stored(step["q_abs"], dt)
        self.o_lat, self.o_lat64 = stored(step["o_lat"], dt)
        if with_weights:
            W = synth.weights(w)
            self.W = {}
            self.W64 = {}
            for k, v in W.items():
                self.W[k], self.W64[k] = stored(v, dt)
            self.w_dkv_kr, _ = stored(np.concatenate([W["W_DKV"], W["W_KR"]], axis=1), dt)

    def pool_rows(self):
        """Pool row of every logical row (sequence b, position p) in logical order."""
        out = np.empty(int(self.row_off[-1]), dtype=np.int64)
        for b, L in enumerate(self.lens):
            p = np.arange(L)
            out[self.row_off[b]:self.row_off[b + 1]] = self.table[b, p // 64].astype(np.int64) * 64 + p % 64
        return out

    def seq_rows64(self, b, pool=None):
        """float64 (c, k_r) rows 0..L-1 of sequence b as stored in `pool` (default: this case's)."""
        pool = self.pool if pool is None else pool
        L = int(self.lens[b])
        p = np.arange(L)
        idx = torch.from_numpy(self.table[b, p // 64].astype(np.int64) * 64 + p % 64)
        rows = pool[idx].to(torch.float64).numpy()
        return rows[:, :self.w.d_c], rows[:, self.w.d_c:]

    def to_device(self, device="cuda"):
        d = {}
        d["pool"] = self.pool.to(device)
        d["seqlens"] = torch.from_numpy(self.lens).to(device)
        d["table"] = torch.from_numpy(self.table).to(device)
        d["x"] = self.x.to(device)
        d["q_nope"] = self.q_nope.to(device)
        d["q_rope_raw"] = self.q_rope_raw.to(device)
        d["q_abs"] = self.q_abs.to(device)
        d["o_lat"] = self.o_lat.to(device)
        if hasattr(self, "W"):
            for k, v in self.W.items():
                d[k] = v.to(device)
            d["w_dkv_kr"] = self.w_dkv_kr.to(device)
        return d


def as_stored(a64, dtype: str):
    """The oracle's own value rounded to the storage type the boundary keeps it in (q_abs and o_lat
    are bf16 tensors between calls in a bf16 pipeline). Nothing here comes from the GPU."""
    return torch.from_numpy(np.asarray(a64, np.float64)).to(TORCH_DT[dtype]).to(torch.float64).numpy()


def max_rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.abs(got - ref).max() / max(np.abs(ref).max(), 1e-300))
