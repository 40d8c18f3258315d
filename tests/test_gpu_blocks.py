"""GPU parity of the whole-block moves (copy-on-write copy, swap-out gather,
swap-in scatter) against the oracle's numpy moves, bit for bit, and decode
attention over sequences that forked, diverged by copy-on-write, or were
swapped out and back in. Every call goes through the C ABI.
"""
import numpy as np
import pytest
import torch

from cow_cases import ForkScenario, random_bf16_bits
from gpu_cases import compare

pytestmark = pytest.mark.gpu


def random_caches(rng, n_caches, num_blocks, Hkv, D, dtype, device):
    host = [rng.integers(0, 2 ** 16, size=(num_blocks, 16, Hkv, D), dtype=np.uint16) for _ in range(n_caches)]
    dev = [torch.from_numpy(h.view(np.int16)).to(device).view(dtype) for h in host]
    return host, dev


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def ids_on(device, ids):
    return torch.tensor(list(ids), dtype=torch.int32, device=device)


@pytest.mark.parametrize("Hkv,D,dtype,n_caches,n", [
    (4, 64, torch.bfloat16, 1, 37),
    (8, 128, torch.float16, 3, 300),
    (2, 64, torch.bfloat16, 64, 700),     # one launch over 64 tensors; grid-stride loop taken
    (1, 8, torch.float16, 2, 5),
    (3, 24, torch.bfloat16, 2, 9),        # 144 chunks per block: four-chunk rounds, then a tail of 16
])
def test_block_moves_bit_exact(pkv, oracle_mod, cuda_device, Hkv, D, dtype, n_caches, n):
    rng = np.random.default_rng(n)
    num_blocks = 2 * n + 11
    host, dev = random_caches(rng, n_caches, num_blocks, Hkv, D, dtype, cuda_device)
    perm = rng.permutation(num_blocks)
    src, dst = perm[:n].tolist(), perm[n:2 * n].tolist()          # disjoint sources and destinations
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)

    packed = torch.empty((n_caches, n, 16, Hkv, D), dtype=dtype, device=cuda_device)
    pkv.kv_cache_gather_blocks(packed, dev, ids_on(cuda_device, src), error_flag=flag)
    pkv.kv_cache_copy_blocks(dev, ids_on(cuda_device, src), ids_on(cuda_device, dst), error_flag=flag)
    torch.cuda.synchronize()
    for c in range(n_caches):
        np.testing.assert_array_equal(bits(packed[c]), oracle_mod.gather_blocks(host[c], src))
        np.testing.assert_array_equal(bits(dev[c]), oracle_mod.copy_blocks(host[c], src, dst))

    # scatter the packed blocks into a third set of blocks of fresh caches
    host2, dev2 = random_caches(rng, n_caches, num_blocks, Hkv, D, dtype, cuda_device)
    tgt = rng.permutation(num_blocks)[:n].tolist()
    pkv.kv_cache_scatter_blocks(dev2, packed, ids_on(cuda_device, tgt), error_flag=flag)
    torch.cuda.synchronize()
    for c in range(n_caches):
        np.testing.assert_array_equal(bits(dev2[c]), oracle_mod.scatter_blocks(host2[c], bits(packed[c]), tgt))
    assert int(flag.item()) == 0


def test_block_moves_skip_and_flag_bad_ids(pkv, oracle_mod, cuda_device):
    rng = np.random.default_rng(3)
    num_blocks, Hkv, D = 20, 2, 64
    host, dev = random_caches(rng, 2, num_blocks, Hkv, D, torch.bfloat16, cuda_device)
    flag = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    src, dst = [1, -1, 3, 4], [10, 11, num_blocks, 13]              # pairs 1 and 2 are bad
    pkv.kv_cache_copy_blocks(dev, ids_on(cuda_device, src), ids_on(cuda_device, dst), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == pkv.KV_STATUS_BAD_BLOCK_ID
    for c in range(2):
        np.testing.assert_array_equal(bits(dev[c]), oracle_mod.copy_blocks(host[c], [1, 4], [10, 13]))
    flag.zero_()
    out = torch.zeros((2, 3, 16, Hkv, D), dtype=torch.bfloat16, device=cuda_device)
    pkv.kv_cache_gather_blocks(out, dev, ids_on(cuda_device, [0, 99, 2]), error_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == pkv.KV_STATUS_BAD_BLOCK_ID
    assert not bits(out[:, 1]).any()                                 # the bad entry was not written
    # empty calls are no-ops; misaligned or oversize requests are refused on the host
    pkv.kv_cache_copy_blocks(dev, ids_on(cuda_device, []), ids_on(cuda_device, []))
    with pytest.raises(pkv.KVError):
        pkv.kv_cache_copy_blocks([dev[0]] * 129, ids_on(cuda_device, [0]), ids_on(cuda_device, [1]))
    odd = torch.empty(num_blocks * 16 * Hkv * D + 1, dtype=torch.bfloat16, device=cuda_device)[1:]
    with pytest.raises(pkv.KVError):
        pkv.kv_cache_copy_blocks([odd.view(num_blocks, 16, Hkv, D)], ids_on(cuda_device, [0]),
                                 ids_on(cuda_device, [1]))


class KernelBackend:
    """Cache writes by the library: one copy launch over every layer's K and V, then the append."""

    def __init__(self, pkv, scenario, device):
        self.pkv, self.device = pkv, device
        shape = (scenario.num_blocks, 16, scenario.Hkv, scenario.D)
        nan = torch.full(shape, 0x7FC0, dtype=torch.int16)
        self.c = [[nan.clone().to(device).view(torch.bfloat16) for _ in range(2)] for _ in range(scenario.n_layers)]
        self.flag = torch.zeros(1, dtype=torch.int32, device=device)

    def copy(self, src, dst):
        flat = [t for layer in self.c for t in layer]
        self.pkv.kv_cache_copy_blocks(flat, ids_on(self.device, src), ids_on(self.device, dst), error_flag=self.flag)

    def append(self, layer, slots, k_new, v_new):
        kn = torch.from_numpy(k_new.view(np.int16)).to(self.device).view(torch.bfloat16)
        vn = torch.from_numpy(v_new.view(np.int16)).to(self.device).view(torch.bfloat16)
        self.pkv.kv_cache_append(kn, vn, self.c[layer][0], self.c[layer][1],
                                 torch.from_numpy(slots).to(self.device), error_flag=self.flag)

    def caches(self):
        torch.cuda.synchronize()
        assert int(self.flag.item()) == 0
        return [[bits(t) for t in layer] for layer in self.c]


def test_copy_on_write_decode_matches_oracle(pkv, oracle_mod, cuda_device):
    """Forked sequences diverge through copy-on-write; every view stays exact and decode over
    the shared and copied blocks matches the oracle."""
    Hq = 8
    sc = ForkScenario(pkv, n_seqs=6, num_blocks=160, W=12, n_layers=2, Hkv=2, D=64, seed=11)
    be = KernelBackend(pkv, sc, cuda_device)
    rng = np.random.default_rng(12)
    ws = pkv.make_workspace(len(sc.live), Hq, sc.Hkv, sc.D)
    checked = []

    def attend(s):
        live = [i for i in range(len(s.live)) if s.live[i]]
        if len(checked) > 6 or len(live) < 2:
            return
        tables = s.tables[live].contiguous()
        lens = s.lens[live].contiguous()
        q_bits = random_bf16_bits(rng, (len(live), Hq, s.D))
        q = torch.from_numpy(q_bits.view(np.int16)).to(cuda_device).view(torch.bfloat16)
        for layer in range(s.n_layers):
            out = torch.empty_like(q)
            pkv.paged_attention_decode(out, q, be.c[layer][0], be.c[layer][1], tables.to(cuda_device),
                                       lens.to(cuda_device), 1.0 / np.sqrt(s.D), ws)
            torch.cuda.synchronize()
            ref = oracle_mod.paged_attention_decode(q_bits, bits(be.c[layer][0]), bits(be.c[layer][1]),
                                                    tables.numpy(), lens.numpy(), 1.0 / np.sqrt(s.D))
            compare(out, ref, f"copy-on-write decode, layer {layer}")
        checked.append(len(live))

    sc.run(oracle_mod, be, n_random_steps=50, check_every=5, on_step=attend)
    assert checked and sc.copies_total >= 3
    assert pkv.read_status(ws) == 0


def test_swap_out_and_in_gives_the_same_decode(pkv, oracle_mod, cuda_device):
    """Preempt two sequences: gather their blocks over every layer, copy them to pinned host
    memory, let other data overwrite the blocks, then scatter them into different blocks and
    rewrite the tables. Decode afterwards is bit-identical to decode before."""
    from paged_kv_cache_470_b200 import workloads
    cfg = workloads.small_config(2, batch=6, n_layers=3, ctx_lo=20, ctx_hi=300)
    layout = workloads.draw_layout(cfg, seed=5)
    gen = workloads.device_generator(5, cuda_device)
    caches = [workloads.make_layer_cache(layout.num_blocks + 64, cfg.Hkv, cfg.D, gen, cuda_device)
              for _ in range(cfg.n_layers)]
    flat = [t for kv in caches for t in kv]
    q = torch.randn(cfg.batch, cfg.Hq, cfg.D, generator=gen, device=cuda_device).to(torch.bfloat16)
    tables, lens = layout.block_tables.to(cuda_device), layout.context_lens.to(cuda_device)
    ws = pkv.make_workspace(cfg.batch, cfg.Hq, cfg.Hkv, cfg.D)

    def decode_all(tab):
        outs = []
        for k, v in caches:
            o = torch.empty_like(q)
            pkv.paged_attention_decode(o, q, k, v, tab, lens, cfg.scale, ws)
            outs.append(o)
        torch.cuda.synchronize()
        return outs

    before = decode_all(tables)
    victims = [1, 4]
    ids = {b: layout.block_tables[b, :-(-int(layout.context_lens[b]) // 16)].tolist() for b in victims}
    swapped = {}
    for b in victims:
        staged = torch.empty((len(flat), len(ids[b]), 16, cfg.Hkv, cfg.D), dtype=torch.bfloat16,
                             device=cuda_device)
        pkv.kv_cache_gather_blocks(staged, flat, ids_on(cuda_device, ids[b]))
        host = torch.empty(staged.shape, dtype=staged.dtype, pin_memory=True)
        host.copy_(staged, non_blocking=True)
        swapped[b] = host
    torch.cuda.synchronize()
    for t in flat:                                                   # the freed blocks are reused
        for b in victims:
            t[ids[b]] = torch.randn(len(ids[b]), 16, cfg.Hkv, cfg.D, device=cuda_device).to(torch.bfloat16)
    used = set(int(x) for x in layout.block_tables.flatten().tolist() if x >= 0)
    spare = [i for i in range(layout.num_blocks + 64) if i not in used]
    new_tables = layout.block_tables.clone()
    for b in victims:
        new_ids, spare = spare[:len(ids[b])], spare[len(ids[b]):]
        pkv.kv_cache_scatter_blocks(flat, swapped[b].to(cuda_device, non_blocking=True),
                                    ids_on(cuda_device, new_ids))
        new_tables[b, :len(new_ids)] = torch.tensor(new_ids, dtype=torch.int32)
    after = decode_all(new_tables.to(cuda_device))
    for layer in range(cfg.n_layers):
        assert torch.equal(before[layer].view(torch.int16), after[layer].view(torch.int16)), layer
        ref = oracle_mod.paged_attention_decode(q.cpu(), caches[layer][0].cpu(), caches[layer][1].cpu(),
                                                new_tables.numpy(), layout.context_lens.numpy(), cfg.scale)
        compare(after[layer], ref, f"after swap-in, layer {layer}")
    assert pkv.read_status(ws) == 0
