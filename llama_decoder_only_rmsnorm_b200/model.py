"""Host-side driver of the C ABI for a whole decoder stack.

Owns the device buffers (through torch: weights are given, the RoPE table,
workspace, KV caches and id/logit outputs are allocated here) and issues one
library call per step: embed -> layer_forward/layer_decode per block ->
lm_head_argmax.  It does no arithmetic of its own.  The layer loop follows
the stack of "Build your own Llama 3 from scratch" 四 (Transformer.forward).
"""
from __future__ import annotations

import torch

from . import binding as B


class Llama3Stack:
    def __init__(self, cfg: dict, layers, out_weights, batch: int, cache_cap: int, max_seq: int,
                 lm_rows: int = 0, device="cuda", rope_len: int | None = None, caches=None, alloc=None):
        """alloc (optional): alloc(shape, dtype, device) -> uninitialised
        tensor, used instead of torch.empty for every buffer this object
        allocates (RoPE table, workspace, caches, outputs, generation state)."""
        self._alloc = alloc
        self.cfg_dict = dict(cfg)
        self.cfg = B.make_config(cfg["dim"], cfg["n_heads"], cfg["n_kv_heads"], cfg["ffn_hidden"],
                                 cfg.get("vocab", 0), cfg["norm_eps"], cfg["rope_theta"], cfg["dtype"])
        self.dtype = torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16
        self.layers = list(layers)
        self.wstructs = [B.make_layer_weights(l) for l in self.layers]
        self.out = out_weights
        self.batch, self.cache_cap, self.max_seq = batch, cache_cap, max_seq
        self.device = device
        hd = cfg["dim"] // cfg["n_heads"]
        self.rope_len = rope_len or max(cache_cap, 1)
        self.rope = self._empty((self.rope_len, hd // 2, 2), torch.float32)
        B.llama3_init_rope_table(self.rope, hd, self.rope_len, cfg["rope_theta"])
        self.lm_rows = max(lm_rows, 1)
        self.ws_bytes = B.llama3_workspace_size(self.cfg, batch, max_seq, self.lm_rows)
        self.ws = self._empty((self.ws_bytes,), torch.uint8)
        if caches is None:
            shape = (batch, cache_cap, cfg["n_kv_heads"], hd)
            caches = [(self._empty(shape, self.dtype).zero_(), self._empty(shape, self.dtype).zero_())
                      for _ in self.layers]
        self.caches = caches
        self.ids_out = self._empty((self.lm_rows,), torch.int32).zero_()

    def _empty(self, shape, dtype):
        if self._alloc is not None:
            return self._alloc(tuple(shape), dtype, self.device)
        return torch.empty(shape, dtype=dtype, device=self.device)

    # -- steps --------------------------------------------------------------
    def embed(self, ids, x, stream=None):
        B.llama3_embed(self.cfg, ids, self.out["tok_embeddings"], x, ids.numel(), stream)

    def forward_layers(self, x, seq, start_pos=0, stream=None, layers=None):
        for i in (range(len(self.layers)) if layers is None else layers):
            kc, vc = self.caches[i]
            B.llama3_layer_forward(self.cfg, self.wstructs[i], self.rope, self.rope_len, x, kc, vc,
                                   self.cache_cap, self.batch, seq, start_pos, self.ws, self.ws_bytes, stream)

    def _decode_chain(self, x, start_pos, positions, stream, layers):
        # Every block in order: one call for the whole step (llama3_decode_step).
        if layers is None or list(layers) == list(range(len(self.layers))):
            B.llama3_decode_step(self.cfg, self.wstructs, self.rope, self.rope_len, x,
                                 [kc for kc, _ in self.caches], [vc for _, vc in self.caches], self.cache_cap,
                                 self.batch, start_pos, positions, self.ws, self.ws_bytes, stream)
            return
        # Any other order: one call per block.  Each block leaves the next
        # block's normalised input in the workspace (llama3_layer_decode_chained);
        # a block is told so only when the call before it, on the same
        # workspace, was the block right before it.
        idx = list(layers)
        for n, i in enumerate(idx):
            kc, vc = self.caches[i]
            nxt = idx[n + 1] if n + 1 < len(idx) else None
            next_norm = self.layers[nxt]["attention_norm"] if nxt is not None and nxt == i + 1 else None
            chained_in = n > 0 and idx[n - 1] == i - 1
            B.llama3_layer_decode_chained(self.cfg, self.wstructs[i], self.rope, self.rope_len, x, kc, vc,
                                          self.cache_cap, self.batch, start_pos, positions, next_norm, chained_in,
                                          self.ws, self.ws_bytes, stream)

    def decode_layers(self, x, start_pos, stream=None, layers=None):
        self._decode_chain(x, start_pos, None, stream, layers)

    def decode_layers_ragged(self, x, positions, max_position, stream=None, layers=None):
        """One decode step where sequence b's token sits at positions[b]
        (int32 device tensor); max_position bounds them all."""
        self._decode_chain(x, max_position, positions, stream, layers)

    def lm_head(self, h, rows, row_stride, logits=None, stream=None):
        B.llama3_lm_head_argmax(self.cfg, self.out["norm"], self.out["output"], h, rows, row_stride,
                                self.ids_out, logits, self.ws, self.ws_bytes, stream)
        return self.ids_out[:rows]

    # -- generation ("Build your own Llama 3 from scratch" 六 generate)
    def generate(self, prompt_ids, n_new, eos_id=None, stream=None, temperature=0.0, top_p=0.9, seed=0,
                 return_logits=False, cuda_graph=False, prompt_lens=None):
        """Prefill the prompts (int32 [batch, S] on the device), then decode
        up to n_new tokens.  temperature <= 0 is greedy (the LM head's argmax);
        otherwise each step's fp32 logits go through llama3_sample_top_p,
        whose draw for sequence b is keyed by the position of the token that
        produced the logits (S - 1 for the first new token, then S, S+1, ...).

        Every decode step is the same sequence of launches with device-side
        state only -- embed the current ids, llama3_layer_decode_ragged per
        block at the device positions, LM head (+ draw) into the current ids,
        llama3_generation_advance -- so with cuda_graph=True it is captured once
        and replayed.  Returns the [batch, n_new] tokens as a host array (and,
        with return_logits, the [n_new, batch, vocab] fp32 logits, not with
        cuda_graph).  With eos_id, llama3_generation_advance keeps a done
        flag per sequence on the device: after a sequence's first eos_id the
        rest of its row is eos_id, and the loop ends as soon as every
        sequence is done (the page's generate stops there too); the host
        reads one flag per step for that.

        prompt_lens (host ints, one per sequence, each <= S): prompts of
        different lengths, left-aligned and padded to S.  The padded prefill
        is exact on each sequence's own rows (causal attention never lets a
        real token see a later padding row); the first LM head reads row
        len[b] - 1 of each sequence, and decoding continues at position
        len[b] (padding K/V in the cache are overwritten before they are
        ever visible)."""
        Bn, S = prompt_ids.shape
        assert Bn == self.batch and S + n_new - 1 <= self.cache_cap
        assert not (cuda_graph and (return_logits or stream is not None))
        D, V = self.cfg_dict["dim"], self.cfg_dict["vocab"]
        dev = self.device
        sampling = temperature > 0
        x = self._empty((Bn, S, D), self.dtype)
        self.embed(prompt_ids, x, stream)
        self.forward_layers(x, S, 0, stream)
        row = (Bn + 3) // 4 * 4            # keeps every history row 16-byte aligned
        stop = eos_id is not None
        hist = self._empty((n_new, row), torch.int32).fill_(eos_id if stop else -1)
        done = self._empty((row + 1,), torch.int32).zero_() if stop else None
        all_done = torch.zeros((1,), dtype=torch.int32).pin_memory() if stop else None
        cur = self._empty((row,), torch.int32)
        lens = [S] * Bn if prompt_lens is None else [int(v) for v in prompt_lens]
        assert len(lens) == Bn and all(1 <= v <= S for v in lens)
        pos = self._empty((Bn,), torch.int32)      # position behind the logits
        pos.copy_(torch.tensor([v - 1 for v in lens], dtype=torch.int32))
        step = self._empty((1,), torch.int32).zero_()
        pick = self._empty((row,), torch.int32)
        keep = return_logits or sampling
        logits = self._empty((n_new if return_logits else 1, Bn, V), torch.float32) if keep else None

        def head(h, stride, k):
            lg = logits[k if return_logits else 0] if keep else None
            B.llama3_lm_head_argmax(self.cfg, self.out["norm"], self.out["output"], h, Bn, stride,
                                    pick if sampling else cur, lg, self.ws, self.ws_bytes, stream)
            if sampling:
                B.llama3_sample_top_p(lg, Bn, V, V, temperature, top_p, seed, 0, cur, stream, positions=pos)
            B.llama3_generation_advance(pos, cur, hist, step, Bn, n_new, row, stream, done=done,
                                        eos_id=eos_id if stop else -1)

        if prompt_lens is None:
            head(x[:, -1], S * D, 0)       # first new token; pos -> S, step -> 1
        else:
            idx = torch.tensor([b * S + v - 1 for b, v in enumerate(lens)], dtype=torch.int32, device=dev)
            last = self._empty((Bn, D), self.dtype)
            B.llama3_gather_rows(self.cfg, x, D, Bn * S, idx, Bn, last, stream)
            head(last, D, 0)
        xd = self._empty((Bn, 1, D), self.dtype)
        max_pos = self.cache_cap - 1

        def decode_step(k):
            B.llama3_embed(self.cfg, cur, self.out["tok_embeddings"], xd, Bn, stream)
            self.decode_layers_ragged(xd, pos, max_pos, stream)
            head(xd, D, k)

        def finished():
            # one int read per step: done[Bn] is set once every sequence has
            # emitted the end token
            if not stop:
                return False
            all_done.copy_(done[Bn:Bn + 1], non_blocking=True)
            (torch.cuda.current_stream() if stream is None else stream).synchronize()
            return bool(all_done.item())

        if finished():
            pass
        elif cuda_graph and n_new > 1:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                decode_step(1)             # warm-up step (also token 1)
            torch.cuda.current_stream().wait_stream(side)
            if n_new > 2 and not finished():
                with torch.cuda.graph(g):
                    decode_step(2)
                for k in range(2, n_new):   # the capture ran nothing: replay steps 2 .. n_new-1
                    if k > 2 and finished():
                        break
                    g.replay()
        else:
            for k in range(1, n_new):
                decode_step(k)
                if finished():
                    break
        self.steps_run = int(step.item())
        toks = hist[:, :Bn].t().cpu().numpy()
        if return_logits:
            return toks, logits.cpu().numpy()
        return toks
