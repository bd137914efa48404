"""block_causal_attention_b200: block-causal GQA attention (QK-Norm + 3D RoPE, mask
given as AttnSlices) for NVIDIA B200 (sm_100a).

The computation lives in libbca.so (C ABI, include/bca.h).  This module only
marshals arguments: PyTorch provides device memory and streams.  There is no CPU
or PyTorch fallback: calls fail loudly when the library or a GPU is missing.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import _abi
from ._abi import BcaError  # noqa: F401

__all__ = ["Plan", "BcaError"]


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


class Plan:
    """A compiled block-causal attention problem (mask, schedule, RoPE tables)."""

    def __init__(self, hq: int, hkv: int, d: int, videos, num_cache_keys: int = 0, slices=None,
                 rope_base=(1e4, 1e4, 1e4), eps: float = 1e-6, o_fp32: bool = False,
                 host_only: bool = False, test_force_timeout: bool = False, fp8: bool = False,
                 no_prologue: bool = False, dq_deterministic: bool = False, cache_k_fp16: bool = False):
        """fp8=True: forward with e4m3 tensor-core operands (BCA_FWD_FP8_E4M3; forward only).
        no_prologue=True: q and k are given post-prologue (BCA_NO_PROLOGUE).
        dq_deterministic=True: dQ by a separate fixed-order pass (BCA_DQ_DETERMINISTIC).
        cache_k_fp16=True: k_cache is fp16 and k_prologue writes fp16 (BCA_CACHE_K_FP16)."""
        flags = (_abi.BCA_O_FP32 if o_fp32 else 0) | (_abi.BCA_PLAN_HOST_ONLY if host_only else 0) | \
            (_abi.BCA_TEST_FORCE_TIMEOUT if test_force_timeout else 0) | (_abi.BCA_FWD_FP8_E4M3 if fp8 else 0) | \
            (_abi.BCA_NO_PROLOGUE if no_prologue else 0) | (_abi.BCA_DQ_DETERMINISTIC if dq_deterministic else 0) | \
            (_abi.BCA_CACHE_K_FP16 if cache_k_fp16 else 0)
        prob, keep = _abi.make_problem(hq, hkv, d, videos, num_cache_keys, slices, rope_base, eps, flags)
        self._lib = _abi.lib()
        self._h = _abi.ctypes.c_void_p()
        rc = self._lib.bca_plan_create(_abi.ctypes.byref(prob), _abi.ctypes.byref(self._h))
        del keep
        _abi.check(rc, "bca_plan_create")
        self.hq, self.hkv, self.d = int(hq), int(hkv), int(d)
        self.o_fp32 = bool(o_fp32)
        self.fp8 = bool(fp8)
        self.cache_k_fp16 = bool(cache_k_fp16)
        self.host_only = bool(host_only)
        self.num_cache_keys = int(num_cache_keys)
        inf = self.info()
        self.nq, self.nk = inf["num_q"], inf["num_k"]
        self.device_index = None
        if not host_only:
            import torch
            self.device_index = torch.cuda.current_device()

    @classmethod
    def from_workload(cls, w, host_only: bool = False, o_fp32: Optional[bool] = None, fp8: bool = False) -> "Plan":
        return cls(w.hq, w.hkv, w.d, w.videos_array(), w.num_cache_keys, w.slices_array(),
                   w.rope_base, w.eps, w.o_fp32 if o_fp32 is None else o_fp32, host_only, fp8=fp8)

    def update_positions(self, videos, stream=None) -> None:
        """Move the videos' start frames (t0) of this plan, same geometry otherwise: only the
        RoPE positions and tables are rewritten (a sliding inference window)."""
        import numpy as np
        vid = np.ascontiguousarray(np.asarray(videos, dtype=np.int32).reshape(-1, 5))
        st = None if self.host_only else self._stream(stream)
        rc = self._lib.bca_plan_update_positions(self._h, vid.ctypes.data if len(vid) else None, len(vid), st)
        _abi.check(rc, "bca_plan_update_positions")

    # ------------------------------------------------------------------ host
    def info(self) -> dict:
        inf = _abi.bca_plan_info()
        _abi.check(self._lib.bca_plan_get_info(self._h, _abi.ctypes.byref(inf)), "bca_plan_get_info")
        return {f: getattr(inf, f) for f, _ in inf._fields_}

    def expand_rows(self, r0: int, r1: int) -> np.ndarray:
        out = np.zeros((r1 - r0, self.nk), dtype=np.uint8)
        _abi.check(self._lib.bca_plan_expand_rows(self._h, r0, r1, out.ctypes.data if out.size else None),
                   "bca_plan_expand_rows")
        return out

    def expand_cols(self, k0: int, k1: int) -> np.ndarray:
        """Coverage of keys [k0, k1) from the backward's transposed tables: [k1-k0, Nq]."""
        out = np.zeros((k1 - k0, self.nq), dtype=np.uint8)
        _abi.check(self._lib.bca_plan_expand_cols(self._h, k0, k1, out.ctypes.data if out.size else None),
                   "bca_plan_expand_cols")
        return out

    def workspace_bytes(self, pass_: int = _abi.BCA_PASS_FWD) -> int:
        return int(self._lib.bca_workspace_bytes(self._h, pass_))

    # ------------------------------------------------------------------ device
    def _stream(self, stream):
        import torch
        if stream is None:
            stream = torch.cuda.current_stream()
        return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else stream

    def alloc_workspace(self, pass_: int = _abi.BCA_PASS_FWD):
        import torch
        return torch.empty(max(16, self.workspace_bytes(pass_)), dtype=torch.uint8, device="cuda")

    def fwd(self, q, k, v, k_cache=None, v_cache=None, *, o=None, lse=None, workspace=None,
            q_gain=None, k_gain=None, stream=None):
        """O [Nq, Hq, D] and LSE [Hq, Nq] for bf16 CUDA tensors q [Nq,Hq,D],
        k/v [Nq,Hkv,D] and (if the plan has a cache) k_cache/v_cache [Nc,Hkv,D]."""
        import torch
        if self.host_only:
            raise BcaError(_abi.BCA_ERR_HOST_ONLY_PLAN, "fwd")
        for name, t, rows, heads in (("q", q, self.nq, self.hq), ("k", k, self.nq, self.hkv),
                                     ("v", v, self.nq, self.hkv)):
            if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or \
                    tuple(t.shape) != (rows, heads, self.d):
                raise ValueError(f"{name}: expected contiguous bf16 CUDA tensor of shape "
                                 f"{(rows, heads, self.d)}, got {t.dtype} {tuple(t.shape)}")
        if self.num_cache_keys:
            kdt = torch.float16 if self.cache_k_fp16 else torch.bfloat16
            for name, t, dt in (("k_cache", k_cache, kdt), ("v_cache", v_cache, torch.bfloat16)):
                if t is None or t.dtype != dt or not t.is_contiguous() or \
                        tuple(t.shape) != (self.num_cache_keys, self.hkv, self.d):
                    raise ValueError(f"{name}: expected {dt} [{self.num_cache_keys}, {self.hkv}, {self.d}]")
        dev = q.device
        if o is None:
            o = torch.empty((self.nq, self.hq, self.d), device=dev,
                            dtype=torch.float32 if self.o_fp32 else torch.bfloat16)
        if lse is None:
            lse = torch.empty((self.hq, self.nq), device=dev, dtype=torch.float32)
        if workspace is None:
            workspace = self.alloc_workspace()
        rc = self._lib.bca_fwd(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                               _ptr(q_gain), _ptr(k_gain), _ptr(o), _ptr(lse), _ptr(workspace),
                               self._stream(stream))
        _abi.check(rc, "bca_fwd")
        return o, lse

    def bwd(self, q, k, v, k_cache, v_cache, o, lse, dout, *, dq=None, dk=None, dv=None, dk_cache=None,
            dv_cache=None, workspace=None, q_gain=None, k_gain=None, stream=None, want_cache_grads=True,
            param_grads=False, accumulate=False):
        """Gradients (fp32) w.r.t. q, k, v (new tokens, through QK-Norm + RoPE) and the
        cache; o, lse are the forward's outputs, dout the upstream gradient of O.
        Returns (dq, dk, dv, dk_cache, dv_cache), and with param_grads=True also
        (dq_gain [D], dk_gain [D], drope_base [3]) appended.  accumulate=True adds the five
        gradients into the given (required) arrays."""
        import torch
        if self.host_only:
            raise BcaError(_abi.BCA_ERR_HOST_ONLY_PLAN, "bwd")
        if dout.dtype != torch.bfloat16 or tuple(dout.shape) != (self.nq, self.hq, self.d) or \
                not dout.is_contiguous():
            raise ValueError("dout: expected contiguous bf16 [Nq, Hq, D]")
        dev = q.device
        f32 = torch.float32
        if accumulate and (dq is None or dk is None or dv is None or
                           (self.num_cache_keys and want_cache_grads and (dk_cache is None or dv_cache is None))):
            raise ValueError("accumulate=True needs the gradient arrays to add into")
        dq = torch.empty((self.nq, self.hq, self.d), device=dev, dtype=f32) if dq is None else dq
        dk = torch.empty((self.nq, self.hkv, self.d), device=dev, dtype=f32) if dk is None else dk
        dv = torch.empty((self.nq, self.hkv, self.d), device=dev, dtype=f32) if dv is None else dv
        if self.num_cache_keys and want_cache_grads:
            shp = (self.num_cache_keys, self.hkv, self.d)
            dk_cache = torch.empty(shp, device=dev, dtype=f32) if dk_cache is None else dk_cache
            dv_cache = torch.empty(shp, device=dev, dtype=f32) if dv_cache is None else dv_cache
        if workspace is None:
            workspace = self.alloc_workspace(_abi.BCA_PASS_BWD)
        if not param_grads and not accumulate:
            rc = self._lib.bca_bwd(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(q_gain),
                                   _ptr(k_gain), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                   _ptr(dk_cache), _ptr(dv_cache), _ptr(workspace), self._stream(stream))
            _abi.check(rc, "bca_bwd")
            return dq, dk, dv, dk_cache, dv_cache
        dgq = torch.empty(self.d, device=dev, dtype=f32) if param_grads else None
        dgk = torch.empty(self.d, device=dev, dtype=f32) if param_grads else None
        dbase = torch.empty(3, device=dev, dtype=f32) if param_grads else None
        rc = self._lib.bca_bwd_ex(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(q_gain),
                                  _ptr(k_gain), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                                  _ptr(dk_cache), _ptr(dv_cache), _ptr(dgq), _ptr(dgk), _ptr(dbase),
                                  1 if accumulate else 0, _ptr(workspace), self._stream(stream))
        _abi.check(rc, "bca_bwd_ex")
        out = (dq, dk, dv, dk_cache, dv_cache)
        return out + (dgq, dgk, dbase) if param_grads else out

    def attn_merge(self, o_a, lse_a, o_b, lse_b, *, o=None, lse=None, stream=None):
        """O (this plan's O type) and LSE of the whole problem from two partial attentions
        over disjoint key subsets (fp32 O, LSE [Hq, Nq])."""
        import torch
        if o is None:
            o = torch.empty((self.nq, self.hq, self.d), device=o_a.device,
                            dtype=torch.float32 if self.o_fp32 else torch.bfloat16)
        if lse is None:
            lse = torch.empty((self.hq, self.nq), device=o_a.device, dtype=torch.float32)
        _abi.check(self._lib.bca_attn_merge(self._h, _ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(o),
                                            _ptr(lse), self._stream(stream)), "bca_attn_merge")
        return o, lse

    def k_prologue(self, k, k_gain=None, *, out=None, stream=None):
        """Post-prologue keys (bf16 [Nq, Hkv, D]) of the plan's new tokens."""
        import torch
        if out is None:
            out = torch.empty((self.nq, self.hkv, self.d), device=k.device,
                              dtype=torch.float16 if self.cache_k_fp16 else torch.bfloat16)
        _abi.check(self._lib.bca_k_prologue(self._h, _ptr(k), _ptr(k_gain), _ptr(out), self._stream(stream)),
                   "bca_k_prologue")
        return out

    def k_prologue_bwd(self, k, dk_hat, k_gain=None, *, dk=None, accumulate=False, stream=None):
        """dL/dk (fp32 [Nq, Hkv, D]) from dL/dk_hat through the prologue; added into dk
        when accumulate=True."""
        import torch
        if dk is None:
            dk = torch.zeros((self.nq, self.hkv, self.d), device=k.device, dtype=torch.float32)
        _abi.check(self._lib.bca_k_prologue_bwd(self._h, _ptr(k), _ptr(k_gain), _ptr(dk_hat), _ptr(dk),
                                                1 if accumulate else 0, self._stream(stream)),
                   "bca_k_prologue_bwd")
        return dk

    def profile(self, enable: bool = True) -> None:
        """Bracket every kernel launched for this plan with CUDA events."""
        _abi.check(self._lib.bca_profile_enable(self._h, 1 if enable else 0), "bca_profile_enable")

    def profile_read(self) -> dict:
        """{kernel name: (launches, total device ms)} since the last read."""
        out = {}
        for k, name in _abi.KERNEL_NAMES.items():
            n = _abi.ctypes.c_int64()
            ms = _abi.ctypes.c_double()
            _abi.check(self._lib.bca_profile_read(self._h, k, _abi.ctypes.byref(n), _abi.ctypes.byref(ms)),
                       "bca_profile_read")
            out[name] = (int(n.value), float(ms.value))
        return out

    def status(self, stream=None) -> int:
        return int(self._lib.bca_status(self._h, self._stream(stream)))

    def close(self) -> None:
        if getattr(self, "_h", None) is not None and self._h.value:
            self._lib.bca_plan_destroy(self._h)
            self._h = _abi.ctypes.c_void_p()

    def __enter__(self) -> "Plan":
        return self

    def __exit__(self, *exc) -> None:
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
