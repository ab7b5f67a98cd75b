"""The integer arithmetic that splits one-token work across CTAs.

The stream-K kernels cut the (column tile, list position) pairs, tile-major,
into G contiguous ranges [floor(c*U/G), floor((c+1)*U/G)), U = tiles * n.
Each column tile's result is assembled from the CTAs whose range meets it;
the kernel finds them with closed forms.  This test checks those forms (as
written in the kernel) against brute force, and that every pair is covered
exactly once with at most two segments per CTA.
"""
import itertools


def contributors(U, G, n, t):
    a = (t * n + 1) * G - 1
    b = (t + 1) * n * G - 1
    return max(0, a // U), min(G - 1, b // U)


def segments(U, G, n, c):
    u0, u1 = U * c // G, U * (c + 1) // G
    out = []
    t = u0 // n
    while t * n < u1 and len(out) < 2:
        a, b = max(u0 - t * n, 0), min(u1 - t * n, n)
        if b > a:
            out.append((t, a, b))
        t += 1
    return out


def test_closed_forms_match_brute_force():
    for n_tiles, n, G in itertools.product([1, 2, 3, 8, 11, 24, 148], [1, 2, 7, 154, 2458, 4096],
                                           [1, 3, 74, 148]):
        U = n_tiles * n
        G = min(G, U)  # the planner never launches more CTAs than units
        if n_tiles > G:
            continue
        seen = {}
        for c in range(G):
            segs = segments(U, G, n, c)
            assert 1 <= len(segs) <= 2
            for t, a, b in segs:
                seen.setdefault(t, set()).add(c)
                for pp in range(a, b):
                    key = (t, pp)
                    assert key not in seen, key
                    seen[key] = c
        for t in range(n_tiles):
            assert all((t, pp) in seen for pp in range(n))
            first, last = contributors(U, G, n, t)
            assert seen[t] == set(range(first, last + 1)), (n_tiles, n, G, t)
