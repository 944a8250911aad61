"""B200 (sm_100a) QJL / FQJL 1-bit key sketches for the KV cache.

A thin Python binding over the C ABI in include/qjl.h. It marshals torch
tensors into device pointers and the current CUDA stream and raises on error
statuses. Every step of the hot path runs in the library's CUDA kernels, and
nothing here computes. PyTorch provides device memory and streams only.

Methods (web pages, cited by title and section):
  * QJL abstract (Zandieh, Daliri, Han) on the "Majid Daliri" author page:
    the sign-bit key sketch plus ||k||, and the asymmetric estimator with an
    unquantised JL-projected query.
  * "Fast Quantized Johnson - Lindenstrauss Transforms": D-FQJL and P-FQJL,
    two randomized Hadamard transforms with a Gaussian second diagonal.
  * KIVI abstract on the "Vladimir Braverman" author page: 2-bit per-token
    values, and the decode step that reads the whole cache per token.
"""

import ctypes

import torch

from ._lib import Options, lib

__all__ = ["Projection", "QJLError", "quantize_keys", "project_queries", "scores",
           "quantize_values_2bit", "decode_attention", "decode_workspace_bytes", "PagedCache", "append_keys",
           "append_values_2bit", "scores_paged", "decode_attention_paged", "decode_paged_workspace_bytes",
           "kivi_quantize_keys_2bit", "kivi_key_scores", "device_errors", "prefill_attention", "lib",
           "KINDS"]

KINDS = {"dense": 0, "dfqjl": 1, "pfqjl": 2}
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}
_EXPORT = {"S": 0, "D_r": 1, "perm": 2, "D_g": 3}


class QJLError(RuntimeError):
    def __init__(self, status, where):
        L = lib()
        self.status = status
        msg = L.qjl_last_error_message().decode()
        super().__init__("%s: %s (%s)" % (where, L.qjl_status_string(status).decode(), msg))


def _check(status, where):
    if status != 0:
        raise QJLError(status, where)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t, name):
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def _cuda_rows(t, name):
    """A 2-D CUDA tensor whose rows are contiguous; the row stride is passed as ld."""
    if not (isinstance(t, torch.Tensor) and t.is_cuda):
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dim() != 2 or t.stride(1) != 1 or t.stride(0) < t.shape[1]:
        raise ValueError("%s must be 2-D with contiguous rows" % name)


class Projection:
    """A drawn random map (dense S, D-FQJL or P-FQJL) resident on the current device."""

    def __init__(self, seed, d, m, kind="dense", dither_sigma_rel=0.5, dg_outer=False, s_bf16=True):
        L = lib()
        opt = Options(float(dither_sigma_rel), int(bool(dg_outer)), int(bool(s_bf16)))
        h = ctypes.c_void_p()
        _check(L.qjl_make_projection(int(seed), int(d), int(m), KINDS[kind], ctypes.byref(opt), ctypes.byref(h)),
               "qjl_make_projection")
        self._h = h
        self.seed, self.d, self.m, self.kind = int(seed), int(d), int(m), kind
        self.dither_sigma_rel, self.dg_outer, self.s_bf16 = float(dither_sigma_rel), bool(dg_outer), bool(s_bf16)
        es = ctypes.c_float()
        _check(L.qjl_projection_info(h, None, None, None, ctypes.byref(es)), "qjl_projection_info")
        self.est_scale = es.value

    @property
    def handle(self):
        return self._h

    def export(self, what):
        """Copy a parameter array to a host torch tensor ('S', 'D_r', 'perm', 'D_g')."""
        nb = self.m // self.d
        shape = (self.m, self.d) if what == "S" else (nb, self.d)
        out = torch.empty(shape, dtype=torch.int32 if what == "perm" else torch.float32)
        _check(lib().qjl_projection_export(self._h, _EXPORT[what], _ptr(out), out.numel() * 4),
               "qjl_projection_export")
        return out

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            lib().qjl_destroy_projection(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def quantize_keys(proj, keys, first_token=0, bits=None, norms=None, stream=None):
    """keys [n, d] (fp32 or bf16, CUDA) -> (bits [n, m/32] int32 words, norms [n] fp32)."""
    _cuda(keys, "keys")
    n, d = keys.shape
    if d != proj.d:
        raise ValueError("keys have d=%d, projection has d=%d" % (d, proj.d))
    if bits is None:
        bits = torch.empty((n, proj.m // 32), dtype=torch.int32, device=keys.device)
    if norms is None:
        norms = torch.empty((n,), dtype=torch.float32, device=keys.device)
    _check(lib().qjl_quantize_keys(proj.handle, _ptr(keys), _DTYPES[keys.dtype], n, keys.stride(0),
                                   int(first_token), _ptr(bits), _ptr(norms), _stream(stream)), "qjl_quantize_keys")
    return bits, norms


def project_queries(proj, q, out=None, stream=None):
    """q [nq, d] fp32 (rows contiguous, any row stride) -> S_eff q [nq, m] fp32 (no quantisation)."""
    _cuda_rows(q, "q")
    if q.dtype != torch.float32:
        raise TypeError("q must be float32")
    nq = q.shape[0]
    if out is None:
        out = torch.empty((nq, proj.m), dtype=torch.float32, device=q.device)
    _check(lib().qjl_project_queries(proj.handle, _ptr(q), nq, q.stride(0), _ptr(out), _stream(stream)),
           "qjl_project_queries")
    return out


def scores(proj, bits, norms, sq, out=None, stream=None):
    """bits [G, N, m/32], norms [G, N], sq [G, J, m] -> estimates [G, J, N] fp32."""
    for t, nm in ((bits, "bits"), (norms, "norms"), (sq, "sq")):
        _cuda(t, nm)
    G, N = norms.shape
    J = sq.shape[1]
    if out is None:
        out = torch.empty((G, J, N), dtype=torch.float32, device=norms.device)
    _check(lib().qjl_scores(proj.handle, _ptr(bits), _ptr(norms), G, N, _ptr(sq), J, _ptr(out), _stream(stream)),
           "qjl_scores")
    return out


def quantize_values_2bit(v, codes=None, scale=None, zero=None, stream=None):
    """v [n, d] (fp32 or bf16) -> (codes [n, d/16] int32, scale [n, d/32] fp16, zero [n, d/32] fp16)."""
    _cuda(v, "v")
    n, d = v.shape
    if codes is None:
        codes = torch.empty((n, d // 16), dtype=torch.int32, device=v.device)
    if scale is None:
        scale = torch.empty((n, d // 32), dtype=torch.float16, device=v.device)
    if zero is None:
        zero = torch.empty((n, d // 32), dtype=torch.float16, device=v.device)
    _check(lib().qjl_quantize_values_2bit(_ptr(v), _DTYPES[v.dtype], n, d, _ptr(codes), _ptr(scale), _ptr(zero),
                                          _stream(stream)), "qjl_quantize_values_2bit")
    return codes, scale, zero


def decode_workspace_bytes(groups, q_per_group, N, d):
    return int(lib().qjl_decode_workspace_bytes(groups, q_per_group, N, d))


def decode_attention(proj, bits, norms, codes, scale, zero, sq, softmax_scale, out=None, workspace=None,
                     stream=None):
    """Fused softmax(est * softmax_scale) . V_hat -> out [G, J, d] fp32."""
    for t, nm in ((bits, "bits"), (norms, "norms"), (codes, "codes"), (scale, "scale"), (zero, "zero"),
                  (sq, "sq")):
        _cuda(t, nm)
    G, N = norms.shape
    J = sq.shape[1]
    d = proj.d
    if out is None:
        out = torch.empty((G, J, d), dtype=torch.float32, device=norms.device)
    need = decode_workspace_bytes(G, J, N, d)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=norms.device)
    _check(lib().qjl_decode_attention(proj.handle, _ptr(bits), _ptr(norms), _ptr(codes), _ptr(scale), _ptr(zero),
                                      G, N, _ptr(sq), J, float(softmax_scale), _ptr(out), _ptr(workspace),
                                      workspace.numel() * workspace.element_size(), _stream(stream)),
           "qjl_decode_attention")
    return out


class PagedCache:
    """Caller-side description of a paged cache (pools, block table, lengths), all CUDA tensors.

    bits [P*T, m/32] int32, norms [P*T] fp32, codes [P*T, d/16] int32, scale/zero [P*T, d/32] fp16,
    block_table [G, max_pages] int32, seq_lens [G] int32; T = page_tokens, P = num_pages.
    """

    def __init__(self, page_tokens, block_table, seq_lens, bits, norms, codes=None, scale=None, zero=None):
        self.page_tokens = int(page_tokens)
        self.block_table, self.seq_lens = block_table, seq_lens
        self.bits, self.norms, self.codes, self.scale, self.zero = bits, norms, codes, scale, zero
        self.num_pages = norms.shape[0] // self.page_tokens
        self.groups, self.max_pages = block_table.shape

    def _table(self):
        return (_ptr(self.block_table), int(self.max_pages), self.page_tokens, int(self.num_pages))


def append_keys(proj, cache, keys, positions, stream=None):
    """Sketch keys [G, d] into the cache at positions [G] (int32) of each group."""
    _cuda(keys, "keys")
    G = keys.shape[0]
    _check(lib().qjl_append_keys(proj.handle, _ptr(keys), _DTYPES[keys.dtype], G, keys.stride(0), _ptr(positions),
                                 *cache._table(), _ptr(cache.bits), _ptr(cache.norms), _stream(stream)),
           "qjl_append_keys")


def append_values_2bit(cache, v, positions, stream=None):
    """2-bit values v [G, d] into the cache at positions [G] (int32) of each group."""
    _cuda(v, "v")
    G, d = v.shape
    _check(lib().qjl_append_values_2bit(_ptr(v), _DTYPES[v.dtype], G, d, _ptr(positions), *cache._table(),
                                        _ptr(cache.codes), _ptr(cache.scale), _ptr(cache.zero), _stream(stream)),
           "qjl_append_values_2bit")


def scores_paged(proj, cache, sq, max_len, out=None, stream=None):
    """sq [G, J, m] -> estimates [G, J, max_len] over each group's seq_lens[g] tokens (the rest untouched)."""
    _cuda(sq, "sq")
    G, J = sq.shape[0], sq.shape[1]
    if out is None:
        out = torch.zeros((G, J, max_len), dtype=torch.float32, device=sq.device)
    _check(lib().qjl_scores_paged(proj.handle, _ptr(cache.bits), _ptr(cache.norms), *cache._table(),
                                  _ptr(cache.seq_lens), G, int(max_len), _ptr(sq), J, _ptr(out), _stream(stream)),
           "qjl_scores_paged")
    return out


def decode_paged_workspace_bytes(groups, max_len, d):
    return int(lib().qjl_decode_paged_workspace_bytes(groups, max_len, d))


def decode_attention_paged(proj, cache, sq, max_len, softmax_scale, out=None, workspace=None, stream=None):
    """sq [G, m] (one query per group) -> softmax(est * softmax_scale) . V_hat [G, d] over the paged cache."""
    _cuda(sq, "sq")
    G = sq.shape[0]
    d = proj.d
    if out is None:
        out = torch.empty((G, d), dtype=torch.float32, device=sq.device)
    need = decode_paged_workspace_bytes(G, max_len, d)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=sq.device)
    _check(lib().qjl_decode_attention_paged(proj.handle, _ptr(cache.bits), _ptr(cache.norms), _ptr(cache.codes),
                                            _ptr(cache.scale), _ptr(cache.zero), *cache._table(),
                                            _ptr(cache.seq_lens), G, int(max_len), _ptr(sq), float(softmax_scale),
                                            _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                            _stream(stream)),
           "qjl_decode_attention_paged")
    return out


def kivi_quantize_keys_2bit(keys, codes=None, scale=None, zero=None, stream=None):
    """KIVI per-channel 2-bit keys: keys [G, N, d] -> (codes [G, N, d/16] int32, scale, zero [G, ceil(N/32), d] fp16)."""
    _cuda(keys, "keys")
    G, N, d = keys.shape
    nb = (N + 31) // 32
    if codes is None:
        codes = torch.empty((G, N, d // 16), dtype=torch.int32, device=keys.device)
    if scale is None:
        scale = torch.empty((G, nb, d), dtype=torch.float16, device=keys.device)
    if zero is None:
        zero = torch.empty((G, nb, d), dtype=torch.float16, device=keys.device)
    _check(lib().qjl_kivi_quantize_keys_2bit(_ptr(keys), _DTYPES[keys.dtype], G, N, d, _ptr(codes), _ptr(scale),
                                             _ptr(zero), _stream(stream)), "qjl_kivi_quantize_keys_2bit")
    return codes, scale, zero


def kivi_key_scores(codes, scale, zero, q, out=None, stream=None):
    """<q, k_hat> over KIVI keys: q [G, J, d] fp32 -> [G, J, N] fp32."""
    for t, nm in ((codes, "codes"), (scale, "scale"), (zero, "zero"), (q, "q")):
        _cuda(t, nm)
    G, N = codes.shape[0], codes.shape[1]
    J, d = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty((G, J, N), dtype=torch.float32, device=q.device)
    _check(lib().qjl_kivi_key_scores(_ptr(codes), _ptr(scale), _ptr(zero), G, N, d, _ptr(q), J, _ptr(out),
                                     _stream(stream)), "qjl_kivi_key_scores")
    return out


def device_errors(device=0, clear=True):
    """The per-device error bits the kernels set (synchronises the device); see include/qjl.h."""
    flags = ctypes.c_int(0)
    lib().qjl_device_errors(int(device), int(bool(clear)), ctypes.byref(flags))
    return flags.value


def prefill_attention(proj, bits, norms, codes, scale, zero, sq, softmax_scale, out=None, stream=None):
    """Causal prefill: bits [G, L, m/32], norms [G, L], codes/scale/zero per token, sq [G, L, m] -> out [G, L, d]."""
    for t, nm in ((bits, "bits"), (norms, "norms"), (codes, "codes"), (scale, "scale"), (zero, "zero"), (sq, "sq")):
        _cuda(t, nm)
    G, L = norms.shape
    if out is None:
        out = torch.empty((G, L, proj.d), dtype=torch.float32, device=norms.device)
    _check(lib().qjl_prefill_attention(proj.handle, _ptr(bits), _ptr(norms), _ptr(codes), _ptr(scale), _ptr(zero), G, L,
                                       _ptr(sq), float(softmax_scale), _ptr(out), _stream(stream)),
           "qjl_prefill_attention")
    return out
