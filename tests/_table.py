"""Helpers of the GPU tests that edit a device table in place (to plant a corrupted page id)."""
from __future__ import annotations

import torch

from head_aware_paged_build_b200 import segpaged as S

BAD_PAGE = 5  # device status code: a table page id outside the pool


def page_record_index(layer, b: int, kv: int, page: int) -> int:
    """int32 index, in the device table, of the 16-byte page record of (b, kv)'s page number `page`.

    Found by content: a head's records hold its physical page ids (plan_head_pages) at a
    stride of four words, each followed by the page's first position.
    """
    ids = S.segpaged_plan_head_pages(layer.plan, b, kv)
    seg = S.segpaged_plan_head_segments(layer.plan, b, kv)[0]  # (first position, length, ...)
    words = layer.table.cpu().view(torch.int32).numpy()
    n = min(4, len(ids), -(-seg[1] // 64))  # records of the first segment's pages
    found = [i for i in range(0, len(words) - 4 * n, 4)  # records are 16-byte aligned
             if all(words[i + 4 * t] == ids[t] and words[i + 4 * t + 1] == seg[0] + 64 * t and
                    words[i + 4 * t + 3] == words[i + 3] for t in range(n))]
    assert len(found) == 1, found
    return found[0] + 4 * page


def corrupt(layer, b: int, kv: int, page: int) -> None:
    """Point (b, kv)'s page number `page` far outside the pool."""
    idx = page_record_index(layer, b, kv, page)
    t = layer.table.view(torch.int32)
    t[idx] = 1 << 30
    torch.cuda.synchronize()


def global_head(wl, b: int = 0) -> int:
    return next(kv for kv in range(wl.num_kv_heads) if wl.policy[b * wl.num_kv_heads + kv][0] == "global")
