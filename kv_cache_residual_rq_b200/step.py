"""A looped model's decode step over a device-resident ResidualQuant cache.

One step runs, loop-major like a looped model, one decode-attention call per
(loop, layer): loops 1 .. L-1 read their residual codes, loop L the BF16
reference.  Each call attends over the cached tokens plus the new token's own
BF16 K/V of that loop; the step can end with the append-encode of the new
token into the cache (its L-1 non-final loops against its final loop, every
layer in one call).  Cache contents come from the seeded generator in
`synth` through the library's own encoder.
"""
import torch

from . import synth


def algorithmic_bytes(w, bits, batch=None, ctx=None):
    """HBM bytes one decode call must move: reference K/V, codes, scales, q, out."""
    b = w.batch if batch is None else batch
    t = w.ctx if ctx is None else ctx
    heads_t = b * w.kv_heads * t
    n = 2 * heads_t * w.head_dim * 2
    if bits != 16:
        n += 2 * heads_t * w.head_dim * bits // 8 + 2 * heads_t * (w.head_dim // w.group) * 2
    n += b * w.q_heads * w.head_dim * (2 + 4)
    return n


class DecodeStep:
    """Device-resident cache of every layer plus the per-step inputs.

    Cache arrays are contiguous across layers, [layers][K, V][B][Hkv][T][...],
    so the step's append-encode covers every layer in one call."""

    def __init__(self, w, device):
        import kv_cache_residual_rq_b200 as rq
        self.w, self.rq = w, rq
        L, N, B, H, T, d = w.loops, w.layers, w.batch, w.kv_heads, w.ctx, w.head_dim
        self.shape = rq.make_shape(B, H, T, d, w.group, w.q_heads)
        cache_shape = rq.make_shape(N * 2 * B, H, T, d, w.group)
        self.ref = torch.empty((N, 2, B, H, T, d), dtype=torch.bfloat16, device=device)
        self.codes = [rq.alloc_codes(cache_shape, b, device) for b in w.bits]
        self.scales = [rq.alloc_scales(cache_shape, b, device) for b in w.bits]
        # exact bytes of one (layer, K or V) part: parts are packed back to back
        self.code_bytes = [B * H * T * d * b // 8 for b in w.bits]
        self.scale_bytes = [B * H * T * (d // w.group) * 2 for b in w.bits]
        assert all(n % 16 == 0 for n in self.code_bytes + self.scale_bytes)
        layer_shape = rq.make_shape(B, H, T, d, w.group)
        for layer in range(N):
            for kind in (0, 1):
                r = synth.reference(w, layer, kind, device)
                self.ref[layer, kind].copy_(r)
                loops = [synth.loop_kv(w, layer, kind, l, r) for l in range(1, L)]
                part = layer * 2 + kind
                rq.rq_encode(layer_shape, loops, self.ref[layer, kind], list(w.bits), w.seed,
                             [self._slice(self.codes[l], self.code_bytes[l], part)
                              for l in range(L - 1)],
                             [self._slice(self.scales[l], self.scale_bytes[l], part)
                              for l in range(L - 1)])
                del loops, r
            torch.cuda.empty_cache()
        # per-step inputs: one query per (loop, layer), and the new token's K/V
        # of every loop and layer ([loop][layer][K, V][B][Hkv][1][d])
        self.q = torch.stack([torch.stack([synth.query(w, layer, loop, device)
                                           for layer in range(N)]) for loop in range(1, L + 1)])
        g = torch.Generator(device=device)
        g.manual_seed(w.seed * 31 + 7)
        newref = torch.randn((N, 2, B, H, 1, d), generator=g, device=device)
        self.new_kv = torch.stack(
            [(newref + w.sigma[l] * torch.randn(newref.shape, generator=g, device=device))
             .to(torch.bfloat16) for l in range(L - 1)] + [newref.to(torch.bfloat16)])
        self.append_shape = rq.make_shape(N * 2 * B, H, 1, d, w.group)
        self.out = torch.empty((L, N, B, w.q_heads, d), dtype=torch.float32, device=device)
        self.ws = rq.alloc_workspace(self.shape, device)
        self.ws_bytes = self.ws.numel()
        self.launches_per_step = L * N + 1

    def cache_bytes(self):
        """Bytes of the resident cache (reference rows, codes, scales)."""
        return (self.ref.numel() * 2 + sum(c.numel() for c in self.codes)
                + sum(s.numel() for s in self.scales))

    @staticmethod
    def _slice(buf, nbytes, part):
        return buf[part * nbytes:(part + 1) * nbytes]

    def run(self, stream, timers=None, bufs=None, append=True):
        """One decode step: every (loop, layer) attends over the cache plus the
        new token's BF16 K/V of that loop; then, with `append`, the new token
        is encoded into the cache (the last slot is reused every step, so T
        stays fixed).
        timers: list to append (start, end, bits, calls) per loop segment --
        events only at loop boundaries, so consecutive calls of a loop stay
        back to back and each launch overlaps its predecessor's tail
        (programmatic dependent launch); an event between two launches would
        serialise them.  bufs: (q, new_kv, out) tensors to use instead of the
        step's own (double-buffered end-to-end loop)."""
        rq, w = self.rq, self.w
        st = stream.cuda_stream
        q_all, kv_all, out_all = bufs if bufs is not None else (self.q, self.new_kv, self.out)
        T = w.ctx
        for li in range(w.loops):
            bits = w.bits[li] if li < w.loops - 1 else 16
            ev = None
            if timers is not None:
                ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                ev[0].record(stream)
            for layer in range(w.layers):
                ck = cv = sk = sv = None
                if bits != 16:
                    ck = self._slice(self.codes[li], self.code_bytes[li], 2 * layer)
                    cv = self._slice(self.codes[li], self.code_bytes[li], 2 * layer + 1)
                    sk = self._slice(self.scales[li], self.scale_bytes[li], 2 * layer)
                    sv = self._slice(self.scales[li], self.scale_bytes[li], 2 * layer + 1)
                rq.rq_decode_attention_tail(
                    self.shape, q_all[li, layer], self.ref[layer, 0], self.ref[layer, 1],
                    ck, cv, sk, sv, bits, w.seed, 0.0, kv_all[li, layer, 0],
                    kv_all[li, layer, 1], 1, 1, out_all[li, layer], self.ws, self.ws_bytes, st)
            if ev is not None:
                ev[1].record(stream)
                timers.append((ev[0], ev[1], bits, w.layers))
        if append:
            rq.rq_encode_at(self.append_shape, 1, 0, T, T - 1, list(kv_all[:w.loops - 1]),
                            kv_all[w.loops - 1], list(w.bits), w.seed, self.codes, self.scales,
                            self.ref, st)

    def step_bytes(self):
        """Algorithmic bytes of the step's decode calls."""
        w = self.w
        total = 0
        for li in range(w.loops):
            bits = w.bits[li] if li < w.loops - 1 else 16
            total += w.layers * algorithmic_bytes(w, bits)
        return total
