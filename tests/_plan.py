"""Decoder of the plan buffer written by mla_decode_plan (layout of csrc/plan.h)."""

import numpy as np


def parse_plan(buf: np.ndarray) -> dict:
    w = buf.view(np.int32)
    hdr = dict(magic=int(w[0]) & 0xFFFFFFFF, version=int(w[1]), batch=int(w[2]),
               q_len=int(w[3]), n_h=int(w[4]), num_items=int(w[5]), num_ctas=int(w[6]),
               num_partials=int(w[7]), num_combine=int(w[8]), cta_off=int(w[9]),
               items_off=int(w[10]), combine_off=int(w[11]), max_pages_used=int(w[12]))
    c0 = hdr["cta_off"] // 4
    hdr["cta_begin"] = w[c0: c0 + hdr["num_ctas"] + 1].copy()
    i0 = hdr["items_off"] // 4
    items = w[i0: i0 + 8 * hdr["num_items"]].reshape(-1, 8)
    hdr["items"] = [dict(b=int(r[0]), j=int(r[1]), page_begin=int(r[2]), page_end=int(r[3]),
                         slot=int(r[4]), L=int(r[5]), qpos=int(r[6])) for r in items]
    k0 = hdr["combine_off"] // 4
    comb = w[k0: k0 + 4 * hdr["num_combine"]].reshape(-1, 4)
    hdr["combine"] = [dict(b=int(r[0]), j=int(r[1]), first_slot=int(r[2]), n_parts=int(r[3]))
                      for r in comb]
    return hdr
