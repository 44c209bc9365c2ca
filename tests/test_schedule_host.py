"""Host models of the forward kernel's work-list arithmetic (prefill_kernel.cuh).

The persistent forward kernel hands out work items with `next_item` (a
boustrophedon per head group that starts at the CTA where the previous group
ended, the start carried from group to group) and decodes them with
multiplications instead of divides (`FastDiv`, whose constants `make_fastdiv`
in attn_api.cu computes). These tests restate both in Python and check the
properties the kernel relies on: every item of the list goes to exactly one CTA,
each CTA meets its items in list order, the carried start equals
(group * items per group) mod grid, and the multiply-shift quotient equals the
integer quotient for every dividend the kernel can pass (0 <= n < 2^31).
"""

import random


def next_items(cta, grid, per_group, n_groups):
    """The items (group, index within group) CTA `cta` takes, in order."""
    pg_mod = per_group % grid
    g, k, start = 0, 0, 0
    out = []
    while g < n_groups:
        c = cta - start
        if c < 0:
            c += grid
        i = k * grid + (grid - 1 - c if k & 1 else c)
        if i < per_group:
            k += 1
            out.append((g, i))
            continue
        g += 1
        k = 0
        start += pg_mod
        if start >= grid:
            start -= grid
    return out


def make_fastdiv(d):
    if d <= 1:
        return 0, 0
    l = 0
    while (1 << l) < d:
        l += 1
    return ((1 << (31 + l)) + d - 1) // d, l - 1


def fdiv(n, f):
    m, s = f
    return n if m == 0 else ((n * m) >> 32) >> s


def test_every_item_once_in_list_order():
    rng = random.Random(7)
    for _ in range(200):
        grid = rng.choice([1, 2, 7, 148, 148, 150])
        per_group = rng.randint(1, 700)
        n_groups = rng.randint(1, 9)
        seen = {}
        for cta in range(grid):
            items = next_items(cta, grid, per_group, n_groups)
            flat = [g * per_group + i for g, i in items]
            assert flat == sorted(flat), "a CTA must meet its items in list order"
            for x in flat:
                assert x not in seen, (grid, per_group, n_groups, x)
                seen[x] = cta
        assert sorted(seen) == list(range(per_group * n_groups))


def test_carried_group_start_is_the_modulo():
    for grid in (1, 5, 148):
        for per_group in (1, 3, 147, 148, 149, 1000, 4097):
            pg_mod, start = per_group % grid, 0
            for g in range(40):
                assert start == (g * per_group) % grid
                start += pg_mod
                if start >= grid:
                    start -= grid


def test_group_first_items_rotate_over_the_ctas():
    # group g's first item goes to CTA (g * items per group) mod grid, so the
    # groups' long first items do not all land on CTA 0
    grid, per_group = 148, 256 + 37
    first_cta = {}
    for cta in range(grid):
        for g, i in next_items(cta, grid, per_group, 4):
            if i == 0:
                first_cta[g] = cta
    for g in range(4):
        assert first_cta[g] == (g * per_group) % grid


def test_fastdiv_matches_integer_division():
    rng = random.Random(11)
    divisors = list(range(1, 3000)) + [rng.randrange(1, 2**31) for _ in range(2000)]
    for d in divisors:
        f = make_fastdiv(d)
        assert 0 <= f[0] < 2**32
        for n in [0, 1, d - 1, d, d + 1, 2 * d - 1, 2 * d, 2**31 - 1, 2**31 - 2] + \
                 [rng.randrange(0, 2**31) for _ in range(20)]:
            if 0 <= n < 2**31:
                assert fdiv(n, f) == n // d, (n, d)
