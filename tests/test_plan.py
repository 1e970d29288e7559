"""Contract tests of the host scheduler (per-SM instruction lists and dependency counters), no GPU.

The lists must cover every output row / attention chunk exactly once, every
counter's per-step target must equal the number of its producers, waits may
only point at earlier ops, and a simulation of the counter protocol (each SM
executes its list in order, an instruction runs once its counter reached its
target) must run every instruction to completion: no cyclic wait.
"""
import collections

import numpy as np
import pytest

import fixtures as fx

mk = pytest.importorskip("auto_regressive_decode_b200.mk")

OP_EMBED, OP_QKV, OP_ATTN, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LMHEAD = 1, 2, 3, 4, 5, 6, 7
OP_ROUTER, OP_EXP_GATEUP, OP_EXP_DOWN = 8, 9, 10
ORDER = {OP_EMBED: 0, OP_QKV: 1, OP_ATTN: 2, OP_OPROJ: 3, OP_GATEUP: 4, OP_DOWN: 5, OP_LMHEAD: 6,
         OP_ROUTER: 4, OP_EXP_GATEUP: 4.5, OP_EXP_DOWN: 5}

CASES = [("tiny", 148), ("tiny", 7), ("tiny", 1), ("dense-0.6b", 148), ("dense-8b", 148), ("dense-8b", 132),
         ("moe-128x8", 148), ("moe-128x8", 5)]


def plan_of(name, n_sm, **kw):
    cfg = fx.CONFIGS[name].replace(**kw)
    return cfg, mk.Plan(mk.model_desc(cfg), n_sm)


def rows_of(cfg, op):
    return {OP_QKV: cfg.q_dim + 2 * cfg.kv_dim, OP_OPROJ: cfg.hidden, OP_GATEUP: cfg.ffn_dim, OP_DOWN: cfg.hidden,
            OP_LMHEAD: cfg.vocab, OP_EMBED: cfg.hidden, OP_ROUTER: cfg.n_experts, OP_EXP_DOWN: cfg.hidden}[op]


@pytest.mark.parametrize("name,n_sm", CASES)
def test_rows_and_chunks_covered_once(name, n_sm):
    cfg, p = plan_of(name, n_sm)
    cover = collections.defaultdict(list)
    attn = collections.Counter()
    slots = collections.Counter()
    for row in p.instrs:
        op, layer = p.op(row), p.layer(row)
        if op == OP_ATTN:
            attn[(layer, int(row[4]))] += 1
            assert int(row[5]) == n_sm
        elif op == OP_EXP_GATEUP:
            slots[(layer, int(row[4]))] += 1
            assert int(row[5]) == n_sm
        else:
            cover[(layer, op)].append((int(row[4]), int(row[5])))
            assert 0 < row[5] - row[4] and (op == OP_EMBED or row[5] - row[4] <= 256)
    for (layer, op), segs in cover.items():
        segs.sort()
        assert segs[0][0] == 0 and segs[-1][1] == rows_of(cfg, op)
        assert all(a[1] == b[0] for a, b in zip(segs, segs[1:])), (layer, op)
    # attention: one slot per SM per layer, on that SM; units of one ring stage
    assert set(attn) == {(l, s) for l in range(cfg.n_layers) for s in range(n_sm)}
    assert set(attn.values()) == {1}
    for s in range(n_sm):
        assert all(int(r[4]) == s for r in p.sm_list(s) if p.op(r) == OP_ATTN)
    assert p.chunk == 32768 // (2 * cfg.head_dim) and p.n_chunks == n_sm
    # MoE: one expert gate/up slot per SM per layer
    assert set(slots) == ({(l, s) for l in range(cfg.n_layers) for s in range(n_sm)} if cfg.n_experts else set())
    assert set(slots.values()) <= {1}


@pytest.mark.parametrize("name,n_sm", CASES)
def test_counter_targets_and_wait_order(name, n_sm):
    cfg, p = plan_of(name, n_sm)
    producers = collections.Counter(int(r[3]) for r in p.instrs if int(r[3]) >= 0 and p.op(r) != OP_ATTN)
    merges = collections.Counter()
    op_of_counter = {}
    for r in p.instrs:
        if int(r[3]) >= 0:
            op_of_counter[int(r[3])] = (p.layer(r) if p.op(r) != OP_EMBED else -1, ORDER[p.op(r)])
        if p.op(r) == OP_ATTN:
            merges[int(r[3])] = 0
    group = cfg.n_q_heads // cfg.n_kv_heads
    nhg = group // min(group, 4)
    for c, t in enumerate(p.targets):
        if c in merges:
            assert t == cfg.batch * cfg.n_kv_heads * nhg
        elif c in producers:
            assert t == producers[c], c
    for r in p.instrs:
        w = int(r[1])
        if w < 0:
            assert p.op(r) == OP_EMBED
            continue
        assert int(r[2]) == p.targets[w]
        me = (p.layer(r) if p.op(r) != OP_EMBED else -1, ORDER[p.op(r)])
        assert op_of_counter[w] < me, "waits only on an earlier op"
    # each SM's list is ordered by (layer, op): waits never point forward in a list
    for s in range(n_sm):
        keys = [(p.layer(r) if p.op(r) != OP_EMBED else -1, ORDER[p.op(r)]) for r in p.sm_list(s)]
        assert keys == sorted(keys)


def simulate(p, cfg, order_seed=0, seq_lens=None):
    """Counter protocol on the host: SMs progress in a random order; returns instructions executed.

    An attention slot runs its pieces for this step's lengths; the last piece
    of a (sequence, KV head, head group) row to count bumps the layer's counter."""
    rng = np.random.default_rng(order_seed)
    counters = np.zeros(len(p.targets), dtype=np.int64)
    tickets = collections.Counter()
    pieces = p.attn_pieces(fx.context_lengths(cfg) if seq_lens is None else seq_lens)
    by_slot = collections.defaultdict(list)
    for pc in pieces:
        by_slot[int(pc[0])].append(pc)
    pos = [0] * p.n_sm
    done = 0
    total = len(p.instrs)
    while done < total:
        progressed = False
        for s in rng.permutation(p.n_sm):
            lst = p.sm_list(s)
            while pos[s] < len(lst):
                r = lst[pos[s]]
                w = int(r[1])
                if w >= 0 and counters[w] < int(r[2]):
                    break
                if p.op(r) == OP_ATTN:
                    for pc in by_slot[int(r[4])]:
                        key = (p.layer(r), int(pc[1]), int(pc[2]))
                        tickets[key] += 1
                        if tickets[key] == int(pc[6]):
                            counters[int(r[3])] += 1
                elif int(r[3]) >= 0:
                    counters[int(r[3])] += 1
                pos[s] += 1
                done += 1
                progressed = True
        if not progressed:
            return done
    assert (counters == np.asarray(p.targets)).all()
    return done


@pytest.mark.parametrize("name,n_sm", [("tiny", 148), ("tiny", 3), ("dense-0.6b", 148), ("dense-8b", 148),
                                       ("dense-13b-b8", 148), ("moe-128x8", 148), ("moe-128x8", 3)])
def test_counter_protocol_completes(name, n_sm):
    cfg, p = plan_of(name, n_sm)
    for seed in range(2):
        assert simulate(p, cfg, seed) == len(p.instrs)


def test_weight_bytes_balanced_over_sms():
    cfg, p = plan_of("dense-8b", 148)
    per_sm = np.zeros(148)
    K = {OP_QKV: cfg.hidden, OP_OPROJ: cfg.q_dim, OP_GATEUP: 2 * cfg.hidden, OP_DOWN: cfg.ffn_dim, OP_LMHEAD: cfg.hidden}
    for s in range(148):
        for r in p.sm_list(s):
            if p.op(r) in K:
                per_sm[s] += (int(r[5]) - int(r[4])) * K[p.op(r)] * 2
    assert per_sm.max() / per_sm.mean() < 1.02


def test_fault_injection_hook_makes_an_unsatisfiable_wait(monkeypatch):
    monkeypatch.setenv("MK_FAULT_INJECT", "wait")
    cfg, p = plan_of("tiny", 148)
    first = p.sm_list(0)[0]
    assert int(first[2]) > p.targets[int(first[1])]
    assert simulate(p, cfg) < len(p.instrs)


def test_invalid_and_unsupported_shapes():
    base = fx.CONFIGS["tiny"]
    bad = [base.replace(n_q_heads=3), base.replace(head_dim=96), base.replace(hidden=252)]
    for cfg in bad:
        with pytest.raises(mk.MkError):
            mk.Plan(mk.model_desc(cfg), 148)
    with pytest.raises(mk.MkError):
        mk.Plan(mk.model_desc(base), 0)


@pytest.mark.parametrize("kw,ok", [
    ({"hidden": 8200}, True), ({"ffn_dim": 65544}, True),          # batch 1 streams K in chunks: no width cap
    ({"ffn_dim": 700}, False), ({"hidden": 260}, False),           # widths are multiples of 8
    ({"n_q_heads": 4, "n_kv_heads": 3}, False), ({"n_q_heads": 32, "n_kv_heads": 2}, False),  # group 1/2/4/8
    ({"batch": 8, "ffn_dim": 704}, True), ({"batch": 9, "ffn_dim": 704}, False),
])
def test_documented_shape_limits(kw, ok):
    # the limits include/mk.h states for mk_create (host-side lowering, no GPU)
    cfg = fx.CONFIGS["tiny"].replace(**kw)
    if ok:
        mk.Plan(mk.model_desc(cfg), 8)
    else:
        with pytest.raises(mk.MkError):
            mk.Plan(mk.model_desc(cfg), 8)


def test_batched_shapes_need_64_column_blocks():
    # the tensor-core GEMV views K (hidden, q width, ffn width) as blocks of 64 columns
    base = fx.CONFIGS["tiny"].replace(batch=4)
    with pytest.raises(mk.MkError):
        mk.Plan(mk.model_desc(base), 148)                  # ffn 688
    mk.Plan(mk.model_desc(base.replace(ffn_dim=704)), 148)
    mk.Plan(mk.model_desc(fx.CONFIGS["tiny"]), 148)          # batch 1 reads rows whole: 688 is fine


@pytest.mark.parametrize("name,kw,n_sm", [("dense-13b-b8", {}, 148), ("dense-13b-b8", {}, 132),
                                          ("tiny", {"batch": 4, "ffn_dim": 704}, 148),
                                          ("tiny", {"batch": 4, "ffn_dim": 704}, 5)])
def test_batched_row_ranges_on_box_boundaries(name, kw, n_sm):
    # a TMA box is 8 rows: every batched GEMV instruction starts on a multiple of 8
    # and stays within one of wq | wk | wv; row caps 128 (96 for gate/up)
    cfg, p = plan_of(name, n_sm, **kw)
    qd, kvd = cfg.q_dim, cfg.kv_dim
    for r in p.instrs:
        op = p.op(r)
        if op in (OP_QKV, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LMHEAD):
            r0, r1 = int(r[4]), int(r[5])
            assert r0 % 8 == 0 and r1 > r0
            assert r1 - r0 <= (96 if op == OP_GATEUP else 128)
            assert r1 % 8 == 0 or r1 == rows_of(cfg, op)
    # balanced: no SM streams more than one 8-row box more than the mean per op
    for op in (OP_QKV, OP_DOWN):
        per = collections.Counter()
        for s in range(n_sm):
            for r in p.sm_list(s):
                if p.op(r) == op and p.layer(r) == 0:
                    per[s] += int(r[5]) - int(r[4])
        assert max(per.values()) <= rows_of(cfg, op) / n_sm + 8


def _pieces_reference(seq_lens, rows_per_seq, unit, n_slots):
    """The schedule restated directly: units of every row in row order, dealt in equal runs."""
    owner = []                                   # (b, row, unit) of every global unit
    for b, S in enumerate(seq_lens):
        for r in range(rows_per_seq):
            owner += [(b, r, u) for u in range(S // unit + 1)]
    U = len(owner)
    n = min(n_slots, U)                          # a slot in use holds at least one unit
    out = []
    for j in range(n):
        run = owner[U * j // n:U * (j + 1) // n]
        k = 0
        while k < len(run):
            b, r, ua = run[k]
            e = k
            while e < len(run) and run[e][:2] == (b, r):
                e += 1
            out.append((j, b, r, ua, run[e - 1][2] + 1))
            k = e
    return out


@pytest.mark.parametrize("name,kw,n_sm,lens", [
    ("dense-13b-b8", {}, 148, None),
    ("dense-13b-b8", {}, 148, [0, 0, 0, 0, 0, 0, 0, 4159]),
    ("dense-8b", {}, 148, [4096]),
    ("tiny", {"batch": 5, "ffn_dim": 704}, 7, [0, 1, 127, 128, 140]),
    ("tiny", {"batch": 3, "n_q_heads": 8, "n_kv_heads": 1, "ffn_dim": 704}, 148, [3, 0, 9]),
])
def test_attention_schedule_partition(name, kw, n_sm, lens):
    cfg, p = plan_of(name, n_sm, **kw)
    lens = fx.context_lengths(cfg) if lens is None else np.asarray(lens, dtype=np.int32)
    group = cfg.n_q_heads // cfg.n_kv_heads
    rows_per_seq = cfg.n_kv_heads * (group // min(group, 4))
    pieces = p.attn_pieces(lens)
    # the library's pieces are the restated schedule's
    assert [tuple(int(x) for x in pc[:5]) for pc in pieces] == _pieces_reference(lens, rows_per_seq, p.chunk, n_sm)
    # every unit of every row exactly once; slots' unit counts differ by at most one
    per_slot = collections.Counter()
    covered = collections.defaultdict(list)
    for j, b, r, ua, ub, k, npc in (tuple(int(x) for x in pc) for pc in pieces):
        per_slot[j] += ub - ua
        covered[(b, r)].append((ua, ub, k, npc))
    assert max(per_slot.values(), default=0) - min([per_slot[j] for j in range(n_sm)]) <= 1
    assert set(covered) == {(b, r) for b in range(cfg.batch) for r in range(rows_per_seq)}
    for (b, r), segs in covered.items():
        segs.sort()
        assert segs[0][0] == 0 and segs[-1][1] == int(lens[b]) // p.chunk + 1
        assert all(x[1] == y[0] for x, y in zip(segs, segs[1:]))
        assert [s[2] for s in segs] == list(range(len(segs))) and {s[3] for s in segs} == {len(segs)}
    # the counter protocol completes under these lengths too
    assert simulate(p, cfg, 0, lens) == len(p.instrs)


def test_attention_schedule_rejects_out_of_range_lengths():
    cfg, p = plan_of("tiny", 148)
    with pytest.raises(mk.MkError):
        p.attn_pieces([cfg.max_ctx])


def test_moe_lowering_edges_and_targets():
    # per layer: ... o_proj -> router rows -> one expert gate/up slot per SM -> expert down rows -> next qkv
    cfg, p = plan_of("moe-128x8", 148)
    kinds = collections.defaultdict(list)
    for r in p.instrs:
        kinds[(p.layer(r), p.op(r))].append(r)
    assert not any(op in (OP_GATEUP, OP_DOWN) for (_, op) in kinds)
    sig, n_sig = {}, {}
    for (l, op), rows in kinds.items():
        # one counter per (layer, op); only the last instruction of an SM's share signals it
        sigs = [int(r[3]) for r in rows if int(r[3]) >= 0]
        assert len(set(sigs)) == 1 and all(int(r[3]) in (-1, sigs[0]) for r in rows)
        sig[(l, op)], n_sig[(l, op)] = sigs[0], len(sigs)
    for l in range(cfg.n_layers):
        router, slots, down = kinds[(l, OP_ROUTER)], kinds[(l, OP_EXP_GATEUP)], kinds[(l, OP_EXP_DOWN)]
        assert sum(int(r[5]) - int(r[4]) for r in router) == cfg.n_experts
        assert sum(int(r[5]) - int(r[4]) for r in down) == cfg.hidden
        assert len(slots) == 148 and p.targets[sig[(l, OP_EXP_GATEUP)]] == 148
        assert all(int(r[1]) == sig[(l, OP_OPROJ)] for r in router)
        assert all(int(r[1]) == sig[(l, OP_ROUTER)] and int(r[2]) == n_sig[(l, OP_ROUTER)] for r in slots)
        assert all(int(r[1]) == sig[(l, OP_EXP_GATEUP)] and int(r[2]) == 148 for r in down)
        if l + 1 < cfg.n_layers:
            assert all(int(r[1]) == sig[(l, OP_EXP_DOWN)] and int(r[2]) == n_sig[(l, OP_EXP_DOWN)]
                       for r in kinds[(l + 1, OP_QKV)])


def test_moe_shape_limits():
    base = fx.CONFIGS["tiny"].replace(ffn_dim=0, n_experts=8, top_k=2, expert_ffn_dim=128, batch=4)
    mk.Plan(mk.model_desc(base), 148)
    mk.Plan(mk.model_desc(base.replace(batch=1)), 148)       # MoE at batch 1 runs on the tensor-core kernel
    for bad in (base.replace(top_k=9, n_experts=16), base.replace(top_k=0), base.replace(top_k=9),
                base.replace(expert_ffn_dim=100), base.replace(n_experts=512), base.replace(batch=8, top_k=9, n_experts=16)):
        with pytest.raises(mk.MkError):
            mk.Plan(mk.model_desc(bad), 148)


@pytest.mark.parametrize("name,n_sm", [("dense-8b", 148), ("dense-8b", 132), ("dense-0.6b", 148), ("tiny", 7)])
def test_batch1_gemv_instructions_cover_each_sm_share_in_bounded_pieces(name, n_sm):
    """Batch 1: each SM's rows of an op are one contiguous share, cut into instructions of at most 64
    rows (gate/up: 64 neurons, streamed as a gate group and an up group once above 32), in order."""
    cfg, p = plan_of(name, n_sm)
    for op in (OP_QKV, OP_OPROJ, OP_GATEUP, OP_DOWN, OP_LMHEAD):
        N = {OP_QKV: cfg.q_dim + 2 * cfg.n_kv_heads * cfg.head_dim, OP_OPROJ: cfg.hidden,
             OP_GATEUP: cfg.ffn_dim, OP_DOWN: cfg.hidden, OP_LMHEAD: cfg.vocab}[op]
        layer = cfg.n_layers if op == OP_LMHEAD else 0
        covered = []
        for s in range(n_sm):
            rows = [(int(r[4]), int(r[5])) for r in p.sm_list(s) if p.op(r) == op and p.layer(r) == layer]
            for (a0, b0), (a1, b1) in zip(rows, rows[1:]):
                assert b0 == a1, (op, s)                      # contiguous, in order
            assert all(0 < b - a <= 64 for a, b in rows), (op, s, rows)
            covered += rows
        covered.sort()
        assert covered[0][0] == 0 and covered[-1][1] == N and all(b == a for (_, b), (a, _) in zip(covered, covered[1:]))
    if name == "dense-8b" and n_sm == 148:
        # 14336 neurons: two gate/up instructions of 48-49 neurons per SM
        per_sm = [sum(1 for r in p.sm_list(s) if p.op(r) == OP_GATEUP and p.layer(r) == 0) for s in range(n_sm)]
        assert set(per_sm) == {2}
