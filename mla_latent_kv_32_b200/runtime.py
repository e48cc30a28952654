"""Device-resident MLA decode workloads driven through the C ABI.

A session uploads one workload's tensors to the GPU (PyTorch allocates the
memory), builds the split-KV plan, and runs decode steps as a fixed sequence
of C-ABI calls on one CUDA stream. PyTorch is used for allocation, copies and
streams only; every arithmetic step runs in libmla's kernels.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np
import torch

from . import mla

D_C, D_R, D_NOPE, D_V, ROW, PAGE = mla.D_C, mla.D_R, mla.D_NOPE, mla.D_V, mla.ROW, mla.PAGE
DEFAULT_SCALE = 1.0 / math.sqrt(D_NOPE + D_R)
FP8_ROW = D_C + 2 * D_R      # bytes per FP8 cache row: [512 E4M3 | 64 bf16]
FP8_FILL_CODE = 0x70         # E4M3 128.0: the filler of slots that hold no token


def to_dev_bf16(bits: np.ndarray, device) -> torch.Tensor:
    """uint16 bf16 bit patterns -> device torch.bfloat16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def bf16_to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_dev(arr: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


class _GraphStep:
    """Capture of a session's ``step`` (fixed buffers and plan) in a CUDA graph;
    ``replay(stream)`` then runs the step's library calls as one launch."""

    def capture(self):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self.step(side)
        torch.cuda.current_stream().wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            self.step(side)
        self.graph = g
        return g

    def replay(self, stream):
        with torch.cuda.stream(stream):
            self.graph.replay()


class DecodeSession(_GraphStep):
    """One attention-only decode step per call of ``step()``:

        mla_append_absorb_q (mla_append_fp8_absorb_q with the FP8 cache):
            the cache append (RoPE on the new keys, paged scatter) and the
            absorption (q~ = q^C W^UK, RoPE on q^R, pack [q~ | q^R]) in one
            launch
        mla_decode_attention (split-KV attention + combine)
        mla_out_absorb   (u = W^UV o)
    """

    def __init__(self, inp, device="cuda", num_ctas: int = 0, max_split: int = -1,
                 scale: float = DEFAULT_SCALE, rope_table: Optional[np.ndarray] = None,
                 fp8: bool = False):
        w = inp.w
        self.w = w
        self.fp8 = fp8
        self.device = torch.device(device)
        self.B, self.q_len, self.n_h = w.B, w.q_len, w.n_h
        self.T = w.B * w.q_len
        self.scale = scale
        dev = self.device
        self.lens = inp.lens
        self.num_pages = inp.pool.shape[0]
        self.max_pages = inp.table.shape[1]
        self.cache = None if fp8 else to_dev_bf16(inp.pool, dev)
        self.table = to_dev(inp.table, dev)
        self.q_nope = to_dev_bf16(inp.q_nope.reshape(self.T, -1), dev)
        self.q_pe = to_dev_bf16(inp.q_pe.reshape(self.T, -1), dev)
        self.c_new = to_dev_bf16(inp.c_new.reshape(self.T, D_C), dev)
        self.k_new = to_dev_bf16(inp.k_new.reshape(self.T, D_R), dev)
        self.w_uk = to_dev_bf16(inp.w_uk, dev)
        self.w_uv = to_dev_bf16(inp.w_uv, dev)
        pos = inp.positions.reshape(-1).astype(np.int32)
        self.seq_idx = to_dev(np.repeat(np.arange(self.B, dtype=np.int32), self.q_len), dev)
        self.pos = to_dev(pos, dev)
        self.max_pos = int(inp.lens.max()) if rope_table is None else rope_table.shape[0]
        tab = mla.mla_rope_table(self.max_pos) if rope_table is None else rope_table
        self.rope = to_dev(tab, dev)
        self.plan_host, self.info = mla.mla_decode_plan(inp.lens, self.B, self.q_len, self.n_h,
                                                        num_ctas, max_split)
        self.plan_dev = torch.empty(self.plan_host.nbytes, dtype=torch.uint8, device=dev)
        mla.mla_plan_upload(self.plan_host, self.plan_dev, self.plan_dev.numel())
        self.ws_bytes = int(self.info.workspace_bytes)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.q_full = torch.empty((self.T, self.n_h, ROW), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty((self.T, self.n_h, D_C), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((self.T, self.n_h), dtype=torch.float32, device=dev)
        self.u = torch.empty((self.T, self.n_h * D_V), dtype=torch.bfloat16, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        if fp8:
            self._fp8_pool(inp)

    def _fp8_pool(self, inp):
        """The FP8 cache of this workload: every slot starts as a large
        finite filler (latent code 128.0, scale 1, k^R bf16 64.0); the
        workload's prefix rows [c | k] then enter through the library's own
        FP8 append at their positions (k rotated there), as a prefill would
        write them. The bf16 pool is dropped."""
        dev = self.device
        self.cache = None
        self.cache8 = torch.empty((self.num_pages, PAGE, FP8_ROW), dtype=torch.uint8, device=dev)
        self.cache8[:, :, :D_C] = FP8_FILL_CODE
        self.cache8[:, :, D_C:].view(torch.int16).fill_(int(np.uint16(0x4280).view(np.int16)))
        self.scales8 = torch.ones((self.num_pages, PAGE), dtype=torch.float32, device=dev)
        table = inp.table
        rows, seq, pos = [], [], []
        for b in range(self.B):
            n = int(inp.lens[b]) - self.q_len
            if n <= 0:
                continue
            pages = table[b, :(n + PAGE - 1) // PAGE]
            rows.append(inp.pool[pages].reshape(-1, ROW)[:n])
            seq.append(np.full(n, b, np.int32))
            pos.append(np.arange(n, dtype=np.int32))
        if rows:
            r = to_dev_bf16(np.concatenate(rows), dev)
            sq, ps = to_dev(np.concatenate(seq), dev), to_dev(np.concatenate(pos), dev)
            mla.mla_cache_append_fp8(self.cache8, self.scales8, self.num_pages, self.table, self.B,
                                     self.max_pages, sq, ps, r, ROW, r[:, D_C:], ROW, self.rope,
                                     self.max_pos, r.shape[0], self.status)
            torch.cuda.synchronize(dev)
            del r, sq, ps

    # the four calls of one step ------------------------------------------
    def append(self, stream=None):
        if self.fp8:
            mla.mla_cache_append_fp8(self.cache8, self.scales8, self.num_pages, self.table,
                                     self.B, self.max_pages, self.seq_idx, self.pos, self.c_new,
                                     D_C, self.k_new, D_R, self.rope, self.max_pos, self.T,
                                     self.status, stream)
            return
        mla.mla_cache_append(self.cache, self.num_pages, self.table, self.B, self.max_pages,
                             self.seq_idx, self.pos, self.c_new, D_C, self.k_new, D_R, self.rope,
                             self.max_pos, self.T, self.status, stream)

    def absorb(self, stream=None):
        mla.mla_absorb_q(self.q_nope, self.n_h * D_NOPE, self.q_pe, self.n_h * D_R, self.w_uk,
                         self.pos, self.rope, self.max_pos, self.T, self.n_h, self.q_full,
                         self.status, stream)

    def attend(self, stream=None, lse=True):
        if self.fp8:
            mla.mla_decode_attention_fp8(self.q_full, self.cache8, self.scales8, self.num_pages,
                                         self.table, self.max_pages, self.B, self.q_len,
                                         self.n_h, self.scale, self.plan_host, self.plan_dev,
                                         self.workspace, self.ws_bytes, self.o,
                                         self.lse if lse else None, self.status, stream)
            return
        mla.mla_decode_attention(self.q_full, self.cache, self.num_pages, self.table,
                                 self.max_pages, self.B, self.q_len, self.n_h, self.scale,
                                 self.plan_host, self.plan_dev, self.workspace, self.ws_bytes,
                                 self.o, self.lse if lse else None, self.status, stream)

    def expand(self, stream=None):
        mla.mla_out_absorb(self.o, self.w_uv, self.T, self.n_h, self.u, self.n_h * D_V, stream)

    def append_absorb(self, stream=None):
        """append + absorb in one launch."""
        if self.fp8:
            mla.mla_append_fp8_absorb_q(self.cache8, self.scales8, self.num_pages, self.table,
                                        self.B, self.max_pages, self.seq_idx, self.pos,
                                        self.c_new, D_C, self.k_new, D_R, self.T, self.q_nope,
                                        self.n_h * D_NOPE, self.q_pe, self.n_h * D_R, self.w_uk,
                                        self.pos, self.rope, self.max_pos, self.T, self.n_h,
                                        self.q_full, self.status, stream)
            return
        mla.mla_append_absorb_q(self.cache, self.num_pages, self.table, self.B, self.max_pages,
                                self.seq_idx, self.pos, self.c_new, D_C, self.k_new, D_R, self.T,
                                self.q_nope, self.n_h * D_NOPE, self.q_pe, self.n_h * D_R,
                                self.w_uk, self.pos, self.rope, self.max_pos, self.T, self.n_h,
                                self.q_full, self.status, stream)

    def step(self, stream=None):
        self.append_absorb(stream)
        self.attend(stream)
        self.expand(stream)

    def read_status(self) -> int:
        return mla.mla_read_status(self.status, clear=True)

    # e2e: per-step inputs from pinned host memory, result back to host ----
    def io_inputs(self):
        """Device tensors a step reads that come from the host each step."""
        return [self.q_nope, self.q_pe, self.c_new, self.k_new]

    def pinned_step_buffers(self):
        """Pinned host copies of the per-step inputs and of the result."""
        ins = [self.q_nope, self.q_pe, self.c_new, self.k_new]
        host_in = [t.cpu().pin_memory() for t in ins]
        host_out = torch.empty(self.u.shape, dtype=self.u.dtype).pin_memory()
        return ins, host_in, host_out

    @staticmethod
    def step_io_bytes(ins, host_out) -> tuple:
        return (sum(t.numel() * t.element_size() for t in ins),
                host_out.numel() * host_out.element_size())


def capture_io_step(sess, host_in, host_out):
    """Record one end-to-end step of ``sess`` in a CUDA graph: the upload of
    the step's inputs from pinned host memory (``host_in``, matching
    ``sess.io_inputs()``), the library calls of the step, and the download of
    the result ``u`` into pinned ``host_out``. One replay runs all of it."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())

    def body():
        for d, h in zip(sess.io_inputs(), host_in):
            d.copy_(h, non_blocking=True)
        sess.step(side)
        host_out.copy_(sess.u, non_blocking=True)

    with torch.cuda.stream(side):
        body()                                    # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        body()
    return g


def run_e2e_graphs(graphs, streams, steps):
    """Steps 0..steps-1: step k replays graphs[k % n] on streams[k % n]; each
    graph holds one session's upload, compute and download, so the sessions'
    copies overlap each other's compute. Returns the host seconds spent
    enqueueing."""
    import time
    n = len(graphs)
    t0 = time.perf_counter()
    for k in range(steps):
        with torch.cuda.stream(streams[k % n]):
            graphs[k % n].replay()
    return time.perf_counter() - t0


class LayerSession(_GraphStep):
    """A whole MLA decode layer from hidden states:

        [c^Q =] h W_DQ^T ; [q^C | q^R] = (c^Q or h) [W_UQ|W_QR]^T   (mla_gemm_bf16)
        [c^KV | k^R] = h [W_DKV|W_KR]^T                              (mla_gemm_bf16)
        mla_cache_append, mla_absorb_q, mla_decode_attention, mla_out_absorb
        out = u W_O^T (float32)                                      (mla_gemm_bf16)

    The rows of h that are queries must be the last B*q_len rows.
    """

    def __init__(self, inp, device="cuda", num_ctas: int = 0, max_split: int = -1,
                 scale: float = DEFAULT_SCALE, folded: bool = False):
        w = inp.w
        self.w = w
        self.folded = folded
        dev = self.device = torch.device(device)
        self.B, self.q_len, self.n_h = w.B, w.q_len, w.n_h
        self.Tq = w.B * w.q_len
        self.T = inp.h.shape[0]
        assert np.array_equal(inp.query_tok, np.arange(self.T - self.Tq, self.T))
        self.scale = scale
        self.hidden = w.hidden
        self.q_lora = w.q_lora
        W = inp.weights
        self.lens = inp.lens
        self.num_pages = inp.pool.shape[0]
        self.max_pages = inp.table.shape[1]
        self.cache = to_dev_bf16(inp.pool, dev)
        self.table = to_dev(inp.table, dev)
        self.h = to_dev_bf16(inp.h, dev)
        if self.q_lora:
            self.w_dq = to_dev_bf16(W["w_dq"], dev)
            self.w_qcat = to_dev_bf16(np.concatenate([W["w_uq"], W["w_qr"]], 0), dev)
        else:
            self.w_qcat = to_dev_bf16(np.concatenate([W["w_q"], W["w_qr"]], 0), dev)
        self.w_kvcat = to_dev_bf16(np.concatenate([W["w_dkv"], W["w_kr"]], 0), dev)
        self.w_uk = to_dev_bf16(W["w_uk"], dev)
        self.w_uv = to_dev_bf16(W["w_uv"], dev)
        self.w_o = to_dev_bf16(W["w_o"], dev)
        self.tok_seq = to_dev(inp.tok_seq, dev)
        self.tok_pos = to_dev(inp.tok_pos, dev)
        self.q_pos = to_dev(inp.tok_pos[self.T - self.Tq:], dev)
        self.max_pos = int(inp.lens.max())
        self.rope = to_dev(mla.mla_rope_table(self.max_pos), dev)
        self.plan_host, self.info = mla.mla_decode_plan(inp.lens, self.B, self.q_len, self.n_h,
                                                        num_ctas, max_split)
        self.plan_dev = torch.empty(self.plan_host.nbytes, dtype=torch.uint8, device=dev)
        mla.mla_plan_upload(self.plan_host, self.plan_dev, self.plan_dev.numel())
        self.ws_bytes = int(self.info.workspace_bytes)
        self.workspace = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=dev)
        nq = self.n_h * (D_NOPE + D_R)
        self.cq = (torch.empty((self.Tq, self.q_lora), dtype=torch.bfloat16, device=dev)
                   if self.q_lora else None)
        self.q = torch.empty((self.Tq, nq), dtype=torch.bfloat16, device=dev)
        self.kv = torch.empty((self.T, ROW), dtype=torch.bfloat16, device=dev)
        self.q_full = torch.empty((self.Tq, self.n_h, ROW), dtype=torch.bfloat16, device=dev)
        self.o = torch.empty((self.Tq, self.n_h, D_C), dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty((self.Tq, self.n_h), dtype=torch.float32, device=dev)
        self.u = torch.empty((self.Tq, self.n_h * D_V), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((self.Tq, self.hidden), dtype=torch.float32, device=dev)
        self.gemm_ws = None
        self._gemm_ws()   # allocated here, not during a step
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        if folded:
            self._fold(W)

    def _fold(self, W):
        """Folded weights, computed once by the library: W~QK (query input ->
        latent query per head) and W~O (latent outputs -> layer output); the
        step then skips the content query, mla_out_absorb and u."""
        dev, n_h = self.device, self.n_h
        self.q_in = self.q_lora or self.hidden
        w_up = to_dev_bf16(W["w_uq"] if self.q_lora else W["w_q"], dev)
        self.w_qr = to_dev_bf16(W["w_qr"], dev)
        self.w_qk_f = torch.empty((n_h * D_C, self.q_in), dtype=torch.bfloat16, device=dev)
        self.w_o_f = torch.empty((self.hidden, n_h * D_C), dtype=torch.bfloat16, device=dev)
        ws = torch.empty(mla.mla_fold_qk_workspace_bytes(n_h), dtype=torch.uint8, device=dev)
        mla.mla_fold_qk(w_up, self.q_in, self.q_in, self.w_uk, n_h, self.w_qk_f, ws, ws.numel())
        mla.mla_fold_o(self.w_o, n_h * D_V, self.hidden, self.w_uv, n_h, self.w_o_f)
        torch.cuda.synchronize(dev)
        del w_up, ws
        self.q_r = torch.empty((self.Tq, n_h * D_R), dtype=torch.bfloat16, device=dev)

    # the layer's calls one by one (step runs them in this order) -------------
    def _gemm_ws(self):
        # split-K partial-sum workspace shared by the layer's projections (the
        # calls run one after another on one stream)
        if getattr(self, "gemm_ws", None) is None:
            n_h, d, Tq = self.n_h, self.hidden, self.Tq
            q_in = self.q_lora or d
            shapes = [(Tq, n_h * (D_NOPE + D_R), q_in), (self.T, ROW, d), (Tq, d, n_h * D_V),
                      (Tq, n_h * D_R, q_in), (Tq, d, n_h * D_C)]
            if self.q_lora:
                shapes.append((Tq, self.q_lora, d))
            need = max(mla.mla_gemm_bf16_workspace_bytes(*sh) for sh in shapes)
            self.gemm_ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.device)
        return self.gemm_ws

    def _gemm(self, X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K, stream):
        ws = self._gemm_ws()
        mla.mla_gemm_bf16_ws(X, ld_x, W, ld_w, C, ld_c, c_fp32, M, N, K, ws, ws.numel(), stream)

    def project_q(self, stream=None):
        n_h, d = self.n_h, self.hidden
        hq = self.h[self.T - self.Tq:]
        nq = n_h * (D_NOPE + D_R)
        if self.q_lora:
            self._gemm(hq, d, self.w_dq, d, self.cq, self.q_lora, 0, self.Tq, self.q_lora, d,
                       stream)
            self._gemm(self.cq, self.q_lora, self.w_qcat, self.q_lora, self.q, nq, 0, self.Tq, nq,
                       self.q_lora, stream)
        else:
            self._gemm(hq, d, self.w_qcat, d, self.q, nq, 0, self.Tq, nq, d, stream)

    def project_kv(self, stream=None):
        d = self.hidden
        self._gemm(self.h, d, self.w_kvcat, d, self.kv, ROW, 0, self.T, ROW, d, stream)

    def append(self, stream=None):
        kv_pe = self.kv[:, D_C:]
        mla.mla_cache_append(self.cache, self.num_pages, self.table, self.B, self.max_pages,
                             self.tok_seq, self.tok_pos, self.kv, ROW, kv_pe, ROW, self.rope,
                             self.max_pos, self.T, self.status, stream)

    def absorb(self, stream=None):
        n_h = self.n_h
        nq = n_h * (D_NOPE + D_R)
        q_pe = self.q[:, n_h * D_NOPE:]
        mla.mla_absorb_q(self.q, nq, q_pe, nq, self.w_uk, self.q_pos, self.rope, self.max_pos,
                         self.Tq, n_h, self.q_full, self.status, stream)

    def append_absorb(self, stream=None):
        """append (every token entering the layer) + absorb (the query tokens)
        in one launch."""
        n_h = self.n_h
        nq = n_h * (D_NOPE + D_R)
        mla.mla_append_absorb_q(self.cache, self.num_pages, self.table, self.B, self.max_pages,
                                self.tok_seq, self.tok_pos, self.kv, ROW, self.kv[:, D_C:], ROW,
                                self.T, self.q, nq, self.q[:, n_h * D_NOPE:], nq, self.w_uk,
                                self.q_pos, self.rope, self.max_pos, self.Tq, n_h, self.q_full,
                                self.status, stream)

    def attend(self, stream=None):
        mla.mla_decode_attention(self.q_full, self.cache, self.num_pages, self.table,
                                 self.max_pages, self.B, self.q_len, self.n_h, self.scale,
                                 self.plan_host, self.plan_dev, self.workspace, self.ws_bytes,
                                 self.o, self.lse, self.status, stream)

    def expand(self, stream=None):
        n_h = self.n_h
        mla.mla_out_absorb(self.o, self.w_uv, self.Tq, n_h, self.u, n_h * D_V, stream)

    def project_out(self, stream=None):
        n_h, d = self.n_h, self.hidden
        self._gemm(self.u, n_h * D_V, self.w_o, n_h * D_V, self.out, d, 1, self.Tq, d, n_h * D_V,
                   stream)

    # the folded step's own calls ---------------------------------------------
    def project_q_folded(self, stream=None):
        n_h, d = self.n_h, self.hidden
        hq = self.h[self.T - self.Tq:]
        if self.q_lora:
            self._gemm(hq, d, self.w_dq, d, self.cq, self.q_lora, 0, self.Tq, self.q_lora, d,
                       stream)
            x, ld = self.cq, self.q_lora
        else:
            x, ld = hq, d
        self._gemm(x, ld, self.w_qr, ld, self.q_r, n_h * D_R, 0, self.Tq, n_h * D_R, ld, stream)

    def absorb_folded(self, stream=None):
        n_h = self.n_h
        x, ld = (self.cq, self.q_lora) if self.q_lora else (self.h[self.T - self.Tq:], self.hidden)
        mla.mla_absorb_q_folded(x, ld, self.q_in, self.q_r, n_h * D_R, self.w_qk_f, self.q_pos,
                                self.rope, self.max_pos, self.Tq, n_h, self.q_full, self.status,
                                stream)

    def project_out_folded(self, stream=None):
        n_h, d = self.n_h, self.hidden
        self._gemm(self.o, n_h * D_C, self.w_o_f, n_h * D_C, self.out, d, 1, self.Tq, d, n_h * D_C,
                   stream)

    def step(self, stream=None):
        if self.folded:
            self.project_q_folded(stream)
            self.project_kv(stream)
            self.append(stream)
            self.absorb_folded(stream)
            self.attend(stream)
            self.project_out_folded(stream)
            return
        self.project_q(stream)
        self.project_kv(stream)
        self.append_absorb(stream)
        self.attend(stream)
        self.expand(stream)
        self.project_out(stream)

    def read_status(self) -> int:
        return mla.mla_read_status(self.status, clear=True)
