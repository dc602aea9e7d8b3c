"""Per-phase durations of the batch-1 kernel, from its phase trace.

``kie_trace_enable`` / ``kie_trace_read`` (layout in ``include/kie.h``) give, per CTA and
token, globaltimer stamps (ns). Slot 0 is the token's start. Each layer l then has 16 slots
from 1 + 16 l: the ends of its 10 phases (slots 0-9), the end of the down fold's wait for
every CTA's read of the residual (10), the input-ready stamps of the QKV and gate/up phases
(11, 12), and the end of this CTA's attention positions (15; 0 when it owns no unit). After
the layers come the LM head's rows, its barrier and the final argmax, then the consumer
warps' ring waits of the token per weight phase (QKV rows, O fold, gate/up rows, down fold,
LM head) and the producer's total wait for free ring slots (ns). Host-side arithmetic only.
"""
from __future__ import annotations

import numpy as np

LAYER_PHASES = ("qkv_rows", "qkv_epilogue", "barrier_qkv_attn", "attention", "o_fold", "barrier_o_gu",
                "gate_up_rows", "gate_up_epilogue", "down_fold", "barrier_down_next")
LAYER_END = len(LAYER_PHASES) - 1  # slot of the layer's last phase end
RING_PHASES = ("qkv_rows", "o_fold", "gate_up_rows", "down_fold", "lm_head_rows")  # consumer wait slots


def batch1_events(n_layers: int) -> int:
    """Trace slots per token of the batch-1 kernel."""
    return 1 + 16 * n_layers + 3 + len(RING_PHASES) + 1


def batch1_phase_us(trace: np.ndarray, n_layers: int, first_token: int = 1) -> dict:
    """Mean durations (µs) of a layer's phases over CTAs, layers and tokens.

    trace: [cta][token][event] as returned by ``Engine.trace_read``. A phase lasts from the
    end of the one before it; the first phase of layer l starts at the end of layer l-1, so
    layer 0 (which also loads the embedding row) is left out when there are several layers.
    The attention phase is also split, over the CTAs that own a unit, into the positions
    (from the end of the barrier to the CTA's last position) and the publish-and-merge rest.
    Tokens before ``first_token`` are left out when later ones exist.
    """
    x = np.asarray(trace, dtype=np.int64)
    n_cta, n_tok, n_ev = x.shape
    if n_ev != batch1_events(n_layers):
        raise ValueError(f"{n_ev} events per token, expected {batch1_events(n_layers)} for {n_layers} layers")
    toks = range(first_token if n_tok > first_token else 0, n_tok)
    layers = range(1, n_layers) if n_layers > 1 else range(0, 1)
    dur = {p: [] for p in LAYER_PHASES}
    positions, merge, per_layer = [], [], []
    head = {"lm_head_rows": [], "lm_head_barrier": [], "argmax": []}
    nr = len(RING_PHASES)
    ring = {p: [] for p in RING_PHASES}
    producer = []
    for t in toks:
        s = x[:, t, :]
        for l in layers:
            base = 1 + 16 * l
            prev = s[:, base - 16 + LAYER_END] if l > 0 else s[:, 0]  # the end of the previous layer (or the token start)
            for i, p in enumerate(LAYER_PHASES):
                dur[p].append(s[:, base + i] - prev)
                prev = s[:, base + i]
            tu = s[:, base + 15]
            own = tu > 0
            positions.extend((tu - s[:, base + 2])[own])
            merge.extend((s[:, base + 3] - tu)[own])
        eh = 1 + 16 * n_layers
        head["lm_head_rows"].append(s[:, eh] - s[:, eh - 16 + LAYER_END])
        head["lm_head_barrier"].append(s[:, eh + 1] - s[:, eh])
        head["argmax"].append(s[:, eh + 2] - s[:, eh + 1])
        for k, p in enumerate(RING_PHASES):  # per token; the layer phases spread over the layers
            ring[p].append(s[:, n_ev - 1 - nr + k] / (1 if p == "lm_head_rows" else n_layers))
        producer.append(s[:, n_ev - 1])
        if n_layers > 1:
            per_layer.append((s[:, 1 + 16 * (n_layers - 1) + LAYER_END] - s[:, 1 + LAYER_END]) / (n_layers - 1))

    def us(arrays):  # mean over every CTA of every entry, ns -> µs
        return round(float(np.mean(np.concatenate([np.ravel(a) for a in arrays]))) / 1e3, 2)

    out = {p: us(dur[p]) for p in LAYER_PHASES}
    if positions:
        out["attention_positions"] = round(float(np.mean(positions)) / 1e3, 2)
        out["attention_publish_merge"] = round(float(np.mean(merge)) / 1e3, 2)
    out.update({k: us(v) for k, v in head.items()})
    if per_layer:
        out["per_layer"] = us(per_layer)
    # consumer time blocked on weights that had not arrived: per layer (per token for the head)
    out["ring_wait"] = {p: us(v) for p, v in ring.items()}
    out["producer_wait_per_token"] = us(producer)
    out["tokens"] = len(toks)
    out["layers_averaged"] = len(layers)
    return out
