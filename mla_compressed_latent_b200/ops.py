"""Python binding of libmla: the C-ABI calls under the same names, taking torch CUDA tensors.

Argument marshalling only: shapes and dtypes are checked, device pointers and sizes are passed,
and a workspace is taken from torch's caching allocator when the caller gives none. Every step of
the computation runs in the library's CUDA kernels; a failing call raises MlaError.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib as L


class MlaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = L.load()
        super().__init__(f"{fn}: {lib.mla_status_string(status).decode()} (status {status})")
        self.status = status


@dataclass(frozen=True)
class Dims:
    H: int
    D: int
    d_r: int
    d_c: int
    d_v: int
    g: int = 0
    page_size: int = 64
    sm_scale: float = 0.0
    rms_eps: float = 1e-6
    rope_base: float = 10000.0

    def c(self) -> L.MlaDims:
        # sm_scale 0 lets the library use its default, 1/sqrt(D + d_r)
        return L.MlaDims(self.H, self.D, self.d_r, self.d_c, self.d_v, self.g, self.page_size, self.sm_scale,
                         self.rms_eps, self.rope_base)

    @staticmethod
    def of(w) -> "Dims":
        """From any object with the attributes of a workload (H, D, d_r, d_c, d_v, g, ...)."""
        return Dims(w.H, w.D, w.d_r, w.d_c, w.d_v, getattr(w, "g", 0), getattr(w, "page_size", 64),
                    getattr(w, "sm_scale", 0.0), getattr(w, "rms_eps", 1e-6), getattr(w, "rope_base", 10000.0))


_DTYPES = {torch.float32: L.MLA_F32, torch.bfloat16: L.MLA_BF16}


def _dt(t: torch.Tensor) -> int:
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return _DTYPES[t.dtype]


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libmla takes device tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn, rc):
    if rc != L.MLA_OK:
        raise MlaError(fn, rc)


def _i32(t):
    if t.dtype != torch.int32:
        raise TypeError("index tensors are int32")
    return t


@dataclass
class LatentCache:
    """Latent pool [num_pages*64, d_c] + RoPE-key pool [num_pages*64, d_r] (views may interleave)."""
    latent: torch.Tensor
    rope: torch.Tensor
    num_pages: int

    @staticmethod
    def interleaved(num_pages: int, d_c: int, d_r: int, dtype, device="cuda") -> "LatentCache":
        rows = torch.empty(num_pages * 64, d_c + d_r, dtype=dtype, device=device)
        return LatentCache(rows[:, :d_c], rows[:, d_c:], num_pages)

    def c(self) -> L.MlaLatentCache:
        return L.MlaLatentCache(self.latent.data_ptr(), self.latent.stride(0), self.rope.data_ptr(),
                                self.rope.stride(0), self.num_pages)


@dataclass
class GqaCache:
    k: torch.Tensor     # [num_pages*64, g, D]
    v: torch.Tensor     # [num_pages*64, g, d_v]
    rope: torch.Tensor  # [num_pages*64, d_r]
    num_pages: int

    def c(self) -> L.MlaGqaCache:
        return L.MlaGqaCache(self.k.data_ptr(), self.k.stride(0), self.v.data_ptr(), self.v.stride(0),
                             self.rope.data_ptr(), self.rope.stride(0), self.num_pages)


@dataclass
class LatentCacheFp8:
    """8-bit latent pool: E4M3 codes [num_pages*64, d_c] uint8 + fp32 scales [num_pages*64] + the
    16-bit RoPE-key pool [num_pages*64, d_r]."""
    codes: torch.Tensor
    scales: torch.Tensor
    rope: torch.Tensor
    num_pages: int

    @staticmethod
    def empty_like(cache: "LatentCache") -> "LatentCacheFp8":
        """Code and scale storage for every row of a 16-bit pool, sharing its RoPE keys."""
        rows, d_c = cache.latent.shape
        dev = cache.latent.device
        return LatentCacheFp8(torch.empty(rows, d_c, dtype=torch.uint8, device=dev),
                              torch.empty(rows, dtype=torch.float32, device=dev), cache.rope, cache.num_pages)

    def c(self) -> L.MlaLatentCacheFp8:
        return L.MlaLatentCacheFp8(self.codes.data_ptr(), self.codes.stride(0), self.scales.data_ptr(),
                                   self.rope.data_ptr(), self.rope.stride(0), self.num_pages)


def _workspace(nbytes, device, workspace):
    if nbytes == 0:
        return workspace, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


# ---------------------------------------------------------------------------------------------
def mla_append_cache(dims: Dims, x, w_dkv_kr, gamma, seqlens, block_table, cache: LatentCache,
                     workspace=None, stream=None):
    lib = L.load()
    B, s_q, C = x.shape
    d = dims.c()
    need = lib.mla_append_workspace_size(ctypes.byref(d), B, s_q, C)
    workspace, wsb = _workspace(need, x.device, workspace)
    cc = cache.c()
    rc = lib.mla_append_cache(ctypes.byref(d), _dt(x), B, s_q, _ptr(x), C, _ptr(w_dkv_kr), _ptr(gamma),
                              _ptr(_i32(seqlens)), _ptr(_i32(block_table)), block_table.shape[1], ctypes.byref(cc),
                              _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
    _check("mla_append_cache", rc)


def mla_project_query(dims: Dims, x, w_dq, gamma_q, w_uq, w_qr, q_nope=None, q_rope_raw=None, workspace=None,
                      stream=None):
    """x [B, s_q, C] -> (q_nope [B, s_q, H, D], q_rope_raw [B, s_q, H, d_r]) through
    c_q = RMSNorm(x·W_DQ)·gamma_q (w_dq [C, d_q], w_uq [d_q, H*D], w_qr [d_q, H*d_r])."""
    lib = L.load()
    B, s_q, C = x.shape
    d_q = w_dq.shape[1]
    if q_nope is None:
        q_nope = torch.empty(B, s_q, dims.H, dims.D, dtype=x.dtype, device=x.device)
    if q_rope_raw is None:
        q_rope_raw = torch.empty(B, s_q, dims.H, dims.d_r, dtype=x.dtype, device=x.device)
    d = dims.c()
    need = lib.mla_query_workspace_size(ctypes.byref(d), B, s_q, C, d_q)
    workspace, wsb = _workspace(need, x.device, workspace)
    rc = lib.mla_project_query(ctypes.byref(d), _dt(x), B, s_q, _ptr(x), C, d_q, _ptr(w_dq), _ptr(gamma_q),
                               _ptr(w_uq), _ptr(w_qr), _ptr(q_nope), _ptr(q_rope_raw),
                               _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
    _check("mla_project_query", rc)
    return q_nope, q_rope_raw


def mla_absorb_q(dims: Dims, q_nope, q_rope_raw, w_uk, seqlens, q_abs=None, stream=None):
    lib = L.load()
    B, s_q, H, D = q_nope.shape
    if q_abs is None:
        q_abs = torch.empty(B, s_q, H, dims.d_c + dims.d_r, dtype=q_nope.dtype, device=q_nope.device)
    d = dims.c()
    rc = lib.mla_absorb_q(ctypes.byref(d), _dt(q_nope), B, s_q, _ptr(q_nope), _ptr(q_rope_raw), _ptr(w_uk),
                          _ptr(_i32(seqlens)), _ptr(q_abs), _stream(stream))
    _check("mla_absorb_q", rc)
    return q_abs


def mla_append_cache_absorb_q(dims: Dims, x, w_dkv_kr, gamma, q_nope, q_rope_raw, w_uk, seqlens, block_table,
                              cache: LatentCache, q_abs=None, workspace=None, stream=None):
    """mla_append_cache and mla_absorb_q of one step in one call (their projections share a launch);
    returns q_abs."""
    lib = L.load()
    B, s_q, C = x.shape
    if q_abs is None:
        q_abs = torch.empty(B, s_q, dims.H, dims.d_c + dims.d_r, dtype=q_nope.dtype, device=q_nope.device)
    d = dims.c()
    need = lib.mla_append_workspace_size(ctypes.byref(d), B, s_q, C)
    workspace, wsb = _workspace(need, x.device, workspace)
    cc = cache.c()
    rc = lib.mla_append_cache_absorb_q(ctypes.byref(d), _dt(x), B, s_q, _ptr(x), C, _ptr(w_dkv_kr), _ptr(gamma),
                                       _ptr(q_nope), _ptr(q_rope_raw), _ptr(w_uk), _ptr(_i32(seqlens)),
                                       _ptr(_i32(block_table)), block_table.shape[1], ctypes.byref(cc), _ptr(q_abs),
                                       _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
    _check("mla_append_cache_absorb_q", rc)
    return q_abs


def mla_decode_workspace_size(dims: Dims, dtype, B, s_q, max_pages) -> int:
    d = dims.c()
    return L.load().mla_decode_workspace_size(ctypes.byref(d), _DTYPES[dtype], B, s_q, max_pages)


def mla_decode_absorbed(dims: Dims, q_abs, cache: LatentCache, block_table, seqlens, o_lat=None, lse=None,
                        workspace=None, stream=None, seqlens_host=None):
    """a3 + a4. seqlens_host: optional host copy of seqlens (int32, B values; a numpy array or a CPU
    tensor) that lets the library launch the decode without the split machinery when nothing is
    cut (mla_decode_absorbed_hinted)."""
    lib = L.load()
    B, s_q, H, _ = q_abs.shape
    if o_lat is None:
        o_lat = torch.empty(B, s_q, H, dims.d_c, dtype=q_abs.dtype, device=q_abs.device)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=q_abs.device)
    d = dims.c()
    max_pages = block_table.shape[1]
    need = lib.mla_decode_workspace_size(ctypes.byref(d), _dt(q_abs), B, s_q, max_pages)
    workspace, wsb = _workspace(need, q_abs.device, workspace)
    cc = cache.c()
    if seqlens_host is None:
        rc = lib.mla_decode_absorbed(ctypes.byref(d), _dt(q_abs), B, s_q, _ptr(q_abs), ctypes.byref(cc),
                                     _ptr(_i32(block_table)), max_pages, _ptr(_i32(seqlens)), _ptr(o_lat), _ptr(lse),
                                     _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
        _check("mla_decode_absorbed", rc)
    else:
        host = torch.as_tensor(seqlens_host, dtype=torch.int32).contiguous()
        if host.is_cuda or host.numel() != B:
            raise ValueError("seqlens_host: B int32 values in host memory")
        rc = lib.mla_decode_absorbed_hinted(ctypes.byref(d), _dt(q_abs), B, s_q, _ptr(q_abs), ctypes.byref(cc),
                                            _ptr(_i32(block_table)), max_pages, _ptr(_i32(seqlens)),
                                            ctypes.c_void_p(host.data_ptr()), _ptr(o_lat), _ptr(lse),
                                            _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
        _check("mla_decode_absorbed_hinted", rc)
    return o_lat, lse


def mla_quantize_latent_fp8(dims: Dims, latent, codes, scales, stream=None):
    """Rows of `latent` [rows, d_c] (dtype, rows may be a view of a pool) into E4M3 `codes` [rows, d_c]
    (uint8) and fp32 `scales` [rows]."""
    lib = L.load()
    rows = latent.shape[0]
    d = dims.c()
    rc = lib.mla_quantize_latent_fp8(ctypes.byref(d), _dt(latent), _ptr(latent), latent.stride(0), rows, _ptr(codes),
                                     codes.stride(0), _ptr(scales), _stream(stream))
    _check("mla_quantize_latent_fp8", rc)
    return codes, scales


def mla_decode_absorbed_fp8(dims: Dims, q_abs, cache: LatentCacheFp8, block_table, seqlens, o_lat=None, lse=None,
                            workspace=None, stream=None):
    lib = L.load()
    B, s_q, H, _ = q_abs.shape
    if o_lat is None:
        o_lat = torch.empty(B, s_q, H, dims.d_c, dtype=q_abs.dtype, device=q_abs.device)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=q_abs.device)
    d = dims.c()
    max_pages = block_table.shape[1]
    need = lib.mla_decode_fp8_workspace_size(ctypes.byref(d), B, s_q, max_pages)
    workspace, wsb = _workspace(need, q_abs.device, workspace)
    cc = cache.c()
    rc = lib.mla_decode_absorbed_fp8(ctypes.byref(d), _dt(q_abs), B, s_q, _ptr(q_abs), ctypes.byref(cc),
                                     _ptr(_i32(block_table)), max_pages, _ptr(_i32(seqlens)), _ptr(o_lat), _ptr(lse),
                                     _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
    _check("mla_decode_absorbed_fp8", rc)
    return o_lat, lse


def mla_out_proj(dims: Dims, o_lat, w_uv, out=None, w_o=None, out_model=None, stream=None):
    lib = L.load()
    B, s_q, H, _ = o_lat.shape
    if out is None:
        out = torch.empty(B, s_q, H, dims.d_v, dtype=o_lat.dtype, device=o_lat.device)
    C = 0
    if w_o is not None:
        C = w_o.shape[1]
        if out_model is None:
            out_model = torch.empty(B, s_q, C, dtype=o_lat.dtype, device=o_lat.device)
    d = dims.c()
    rc = lib.mla_out_proj(ctypes.byref(d), _dt(o_lat), B, s_q, _ptr(o_lat), _ptr(w_uv), _ptr(out), _ptr(w_o), C,
                          _ptr(out_model), _stream(stream))
    _check("mla_out_proj", rc)
    return (out, out_model) if w_o is not None else out


def mla_decode_gqla_grouped(dims: Dims, q_nope, q_rope_raw, cache: GqaCache, block_table, seqlens, out=None,
                            lse=None, workspace=None, stream=None):
    lib = L.load()
    B, s_q, H, _ = q_nope.shape
    if out is None:
        out = torch.empty(B, s_q, H, dims.d_v, dtype=q_nope.dtype, device=q_nope.device)
    if lse is None:
        lse = torch.empty(B, s_q, H, dtype=torch.float32, device=q_nope.device)
    d = dims.c()
    max_pages = block_table.shape[1]
    need = lib.mla_gqla_workspace_size(ctypes.byref(d), _dt(q_nope), B, s_q, max_pages)
    workspace, wsb = _workspace(need, q_nope.device, workspace)
    cc = cache.c()
    rc = lib.mla_decode_gqla_grouped(ctypes.byref(d), _dt(q_nope), B, s_q, _ptr(q_nope), _ptr(q_rope_raw),
                                     ctypes.byref(cc), _ptr(_i32(block_table)), max_pages, _ptr(_i32(seqlens)),
                                     _ptr(out), _ptr(lse), _ptr(workspace) if workspace is not None else None, wsb,
                                     _stream(stream))
    _check("mla_decode_gqla_grouped", rc)
    return out, lse


def mla_append_gqa_cache(dims: Dims, x, w_dkv_kr, gamma, w_uk_g, w_uv_g, seqlens, block_table, cache: GqaCache,
                         workspace=None, stream=None):
    """Append this step's tokens to the expanded GQA cache: k_r and, per group, K = W_UK[g]·c and
    V = c·W_UV[g] of c = RMSNorm(x·W_DKV) (x [B, s_q, C], w_uk_g [g, D, d_c], w_uv_g [g, d_c, d_v])."""
    lib = L.load()
    B, s_q, C = x.shape
    d = dims.c()
    need = lib.mla_gqa_append_workspace_size(ctypes.byref(d), B, s_q, C)
    workspace, wsb = _workspace(need, x.device, workspace)
    cc = cache.c()
    rc = lib.mla_append_gqa_cache(ctypes.byref(d), _dt(x), B, s_q, _ptr(x), C, _ptr(w_dkv_kr), _ptr(gamma),
                                  _ptr(w_uk_g), _ptr(w_uv_g), _ptr(_i32(seqlens)), _ptr(_i32(block_table)),
                                  block_table.shape[1], ctypes.byref(cc),
                                  _ptr(workspace) if workspace is not None else None, wsb, _stream(stream))
    _check("mla_append_gqa_cache", rc)


def mla_preabsorb_out_weights(dims: Dims, w_uv, w_o, w_uvo=None, stream=None):
    """W_UVO [H, d_c, C] with W_UVO[h] = W_UV[h] · W_O[h*d_v:(h+1)*d_v] (w_uv [H, d_c, d_v], w_o [H*d_v, C])."""
    lib = L.load()
    C = w_o.shape[1]
    if w_uvo is None:
        w_uvo = torch.empty(dims.H, dims.d_c, C, dtype=w_uv.dtype, device=w_uv.device)
    d = dims.c()
    rc = lib.mla_preabsorb_out_weights(ctypes.byref(d), _dt(w_uv), _ptr(w_uv), _ptr(w_o), C, _ptr(w_uvo),
                                       _stream(stream))
    _check("mla_preabsorb_out_weights", rc)
    return w_uvo


def mla_out_proj_preabsorbed(dims: Dims, o_lat, w_uvo, out_model=None, stream=None):
    """out_model [B, s_q, C] = concat_h(o_lat[..., h, :]) · W_UVO (o_lat [B, s_q, H, d_c], w_uvo [H, d_c, C])."""
    lib = L.load()
    B, s_q, H, _ = o_lat.shape
    C = w_uvo.shape[-1]
    if out_model is None:
        out_model = torch.empty(B, s_q, C, dtype=o_lat.dtype, device=o_lat.device)
    d = dims.c()
    rc = lib.mla_out_proj_preabsorbed(ctypes.byref(d), _dt(o_lat), B, s_q, _ptr(o_lat), _ptr(w_uvo), C,
                                      _ptr(out_model), _stream(stream))
    _check("mla_out_proj_preabsorbed", rc)
    return out_model


def mla_check_status(stream=None) -> int:
    return L.load().mla_check_status(_stream(stream))


def mla_status_string(status: int) -> str:
    return L.load().mla_status_string(status).decode()


def mla_build_info() -> str:
    return L.load().mla_build_info().decode()


def mla_launch_count() -> int:
    return int(L.load().mla_launch_count())
