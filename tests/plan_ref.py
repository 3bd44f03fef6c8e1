"""Host restatement of the split planner, used to check the device plan bit for bit.

The pages of all requests, end to end in request order, are cut into G equal shares
(share g = pages [floor(total*g/G), floor(total*(g+1)/G))); a request is cut wherever
a share boundary falls strictly inside it.  Returns the per-group first-segment index,
the per-request first-segment index and the segment list (b, tile_begin, tile_end,
split flag).
"""
import numpy as np

PAGE = 64


def num_groups_for(num_sms, nqb):
    return max(1, num_sms // nqb)


def plan(seq_lens, G):
    tiles = [(int(t) + PAGE - 1) // PAGE for t in seq_lens]
    total = sum(tiles)
    cut = lambda g: total * g // G
    segs, req_seg, group_begin = [], [], [0] * (G + 1)
    g = 0
    prefix = 0
    for b, n in enumerate(tiles):
        req_seg.append(len(segs))
        pos, end = prefix, prefix + n
        while pos < end:
            while g < G and cut(g + 1) <= pos:
                g += 1
                group_begin[g] = len(segs)
            e = min(cut(g + 1), end)
            segs.append([b, pos - prefix, e - prefix, 0])
            pos = e
        if len(segs) - req_seg[b] > 1:
            for k in range(req_seg[b], len(segs)):
                segs[k][3] = 1
        prefix = end
    req_seg.append(len(segs))
    while g < G:
        g += 1
        group_begin[g] = len(segs)
    return np.array(group_begin, np.int32), np.array(req_seg, np.int32), np.array(segs, np.int32).reshape(-1, 4)
