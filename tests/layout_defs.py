"""Pure-Python statement of the routing layout, for tiny inputs.

Written as ranks (counting, O(n^2)), not as a sort, so that it does not share
a formulation with the oracle it pins.  Definitions:

* a routed pair (t, k) is valid when e = idx[t][k] is in [0, G) and
  part_of[e] is in [0, E_part);
* exp_row[t][k] = number of valid pairs whose key (p, e, t, k) is smaller;
* expert_offset[e] = rows of the experts that precede e in (p, e) order;
* dedup: D = distinct (t, p); disp_row[t][p] = number of pairs of D with a
  smaller (p, t), or -1.
"""


def py_layout(idx, part_of, G, E, dedup):
    M = len(idx)
    topk = len(idx[0]) if M else 0
    st = 0
    for e in range(G):
        if not (0 <= part_of[e] < E):
            st |= 2
    valid = []
    for t in range(M):
        for k in range(topk):
            e = idx[t][k]
            if not (0 <= e < G):
                st |= 1
                continue
            if not (0 <= part_of[e] < E):
                continue
            valid.append((t, k))

    def key(a):
        e = idx[a[0]][a[1]]
        return (part_of[e], e, a[0], a[1])

    exp_row = [[-1] * topk for _ in range(M)]
    for a in valid:
        exp_row[a[0]][a[1]] = sum(1 for b in valid if key(b) < key(a))
    count = [sum(1 for a in valid if idx[a[0]][a[1]] == e) for e in range(G)]

    def ekey(e):
        p = part_of[e]
        return (p if 0 <= p < E else E, e)

    n = len(valid)
    offset = []
    for e in range(G):
        if 0 <= part_of[e] < E:
            offset.append(sum(count[f] for f in range(G) if ekey(f) < ekey(e)))
        else:
            offset.append(n)
    offset.append(n)

    out = dict(expert_count=count, expert_offset=offset, exp_row=exp_row,
               status=st, R_exp=n)
    if not dedup:
        pc = [sum(count[e] for e in range(G) if part_of[e] == p) for p in range(E)]
        disp_token = [None] * n
        for a in valid:
            disp_token[exp_row[a[0]][a[1]]] = a[0]
        out.update(part_count=pc, disp_token=disp_token, R_disp=n)
    else:
        D = sorted({(a[0], part_of[idx[a[0]][a[1]]]) for a in valid})
        disp_row = [[-1] * E for _ in range(M)]
        for (t, p) in D:
            disp_row[t][p] = sum(1 for (t2, p2) in D if (p2, t2) < (p, t))
        disp_token = [None] * len(D)
        for (t, p) in D:
            disp_token[disp_row[t][p]] = t
        pc = [sum(1 for (t, p2) in D if p2 == p) for p in range(E)]
        e2d = [None] * n
        for a in valid:
            e = idx[a[0]][a[1]]
            e2d[exp_row[a[0]][a[1]]] = disp_row[a[0]][part_of[e]]
        out.update(part_count=pc, disp_token=disp_token, disp_row=disp_row,
                   exp_to_disp=e2d, R_disp=len(D))
    po = [0]
    for p in range(E):
        po.append(po[-1] + out["part_count"][p])
    out["part_offset"] = po
    return out
