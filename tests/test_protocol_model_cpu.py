"""The attention kernel's barrier protocol, checked on the CPU by the
randomised model in protocol_model.py: random problem shapes, item schedules,
masks of bf16 blocks and completion orders run without deadlock, parity
aliasing or a buffer hazard, and planted protocol mistakes are caught."""
import os
import random
import types

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = open(os.path.join(HERE, "protocol_model.py")).read()


def load(src):
    mod = types.ModuleType("protocol_model_variant")
    exec(compile(src, "protocol_model_variant", "exec"), mod.__dict__)
    return mod


def configs(n, seed=12345):
    rng = random.Random(seed)
    for t in range(n):
        G = rng.randint(1, 4)
        yield dict(seed=t, B=1, H=rng.randint(1, 3), T=rng.randint(1, 7), causal=rng.random() < 0.6, G=G,
                   cta=rng.randrange(G), mixed=rng.random() < 0.7,
                   pmask=rng.choice([0.0, 0.1, 0.3, 0.7, 1.0]))


def first_failure(mod, n):
    for cfg in configs(n):
        try:
            mod.Sim(**cfg).run()
        except mod.Err as e:
            return cfg, str(e)
    return None


def test_random_schedules_run_clean():
    assert first_failure(load(SRC), 400) is None


# each planted mistake is a real way to get the protocol wrong
MISTAKES = {
    "K/V stage released after one of its two readers":
        ('s.kv_empty = [Bn(f"kv_empty{i}", 2) for i in range(s.S)]',
         's.kv_empty = [Bn(f"kv_empty{i}", 1) for i in range(s.S)]'),
    "P V issued without waiting for its stage":
        ("                yield from s.wait(s.kv_full[st], gt // S, 'pv kv_full')\n", ""),
    "raw Q buffer never handed back":
        ("                            if qhold is not None:\n"
         "                                s.commit(s.qb_empty)  # the raw Q buffer may be reloaded after the Q K^T so far\n",
         ""),
    "S overwritten before it is read":
        ("                    if last is not None:\n"
         "                        yield from s.wait(s.s_free[last[0]], last[1], 'qk s_free')\n", ""),
    "bf16 P written without its grant":
        ("                    yield from s.wait(s.pb_grant[x], nb, who + ' pb_grant')\n                    nb += 1",
         "                    nb += 1"),
    "raw K released after every bf16 Q K^T":
        ("                        if x == 1 or not bB:\n                            s.commit(s.kb_empty)\n"
         "                            bk += 1",
         "                        s.commit(s.kb_empty)\n                        bk += 1"),
    "S released after half of its readers":
        ('s.s_free = [Bn(f"s_free{i}", 8)', 's.s_free = [Bn(f"s_free{i}", 4)'),
    "O rescaled without waiting for the previous P V":
        ("                if k > 0:\n                    yield from s.wait(s.o_done[x], k - 1, who + ' o_done')",
         "                pass"),
    "ring stage reloaded one phase early":
        ("if g < s.S or test(s.kv_empty[st], g // s.S - 1, 'prod ring'):",
         "if g < s.S + 1 or test(s.kv_empty[st], max(g // s.S - 1, 0), 'prod ring'):"),
}


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name):
    old, new = MISTAKES[name]
    assert SRC.count(old) == 1, name
    assert first_failure(load(SRC.replace(old, new)), 120) is not None, name
