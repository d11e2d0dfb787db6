"""Parity of one decode arithmetic path and split-KV mode over every group size
(run as a subprocess).

The path and the split mode are chosen once per process by the PA_DECODE_PATH
(``cuda_cores`` or ``tensor``) and PA_DECODE_SPLIT (``cta`` or ``warp``)
environment variables, so each combination is checked in a process of its own.
16-bit and 8-bit (E4M3) caches are both covered. Exits non-zero on the first
mismatch against the oracle.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import paged_kv_cache_352_b200 as pa  # noqa: E402
from tests.parity import assert_close, out_to_f64, tensor_bits  # noqa: E402


def case(ctx, hq, hkv, d, dtype, nb, seed):
    g = torch.Generator().manual_seed(seed)
    kc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    vc = torch.randn(nb, hkv, 16, d, generator=g).to(dtype).cuda()
    # plant NaN patterns in every unused slot: outputs must not depend on them
    q = torch.randn(len(ctx), hq, d, generator=g).to(dtype).cuda()
    perm = torch.randperm(nb, generator=g)
    mb = max(-(-c // 16) for c in ctx)
    tables = torch.full((len(ctx), mb), -1, dtype=torch.int32)
    used = 0
    for s, c in enumerate(ctx):
        n = -(-c // 16)
        tables[s, :n] = perm[used:used + n].to(torch.int32)
        last = int(perm[used + n - 1])
        if c % 16:
            kc[last, :, c % 16:] = float("nan")
            vc[last, :, c % 16:] = float("nan")
        used += n
    return q, kc, vc, tables.cuda(), torch.tensor(ctx, dtype=torch.int32).cuda()


def main():
    from oracle.attention import paged_decode
    ctx = [1, 9, 16, 33, 250, 1100]
    for G in (1, 2, 4, 8):
        for d in (64, 128):
            for dtype, name in ((torch.float16, "f16"), (torch.bfloat16, "bf16")):
                hkv = 2
                q, kc, vc, tables, cl = case(ctx, G * hkv, hkv, d, dtype, 256, G * 131 + d)
                for pt in (0, 16, 64, 512):
                    out = torch.empty_like(q)
                    err = torch.zeros(1, dtype=torch.int32, device="cuda")
                    ws = pa.decode_workspace(len(ctx), G * hkv, hkv, d, max(ctx), pt)
                    pa.pa_paged_decode(out, q, kc, vc, tables, cl, max(ctx), 0.125, pt, ws, err)
                    torch.cuda.synchronize()
                    assert err.item() == 0, err.item()
                    ref = paged_decode(tensor_bits(q), tensor_bits(kc), tensor_bits(vc),
                                       tables.cpu().numpy(), cl.cpu().numpy(), 0.125, name)
                    assert_close(out_to_f64(out, name), ref,
                                 f"{os.environ.get('PA_DECODE_PATH')} "
                                 f"{os.environ.get('PA_DECODE_SPLIT')} G{G} d{d} {name} pt{pt}")
                fp8_case(ctx, G, hkv, d, dtype, name, tables, cl)
    print("ok")


def fp8_case(ctx, G, hkv, d, dtype, name, tables, cl):
    """The same tables over E4M3 caches of random codes, NaN codes past each context."""
    import numpy as np
    from oracle import fp8 as F
    nb = 256
    g = torch.Generator().manual_seed(G * 7 + d)
    codes = torch.randint(0, 256, (2, nb, hkv, 16, d), generator=g, dtype=torch.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x2C
    tab = tables.cpu().numpy()
    for s, c in enumerate(ctx):
        if c % 16:
            codes[:, int(tab[s, c // 16]), :, c % 16:, :] = 0x7F
    kc, vc = codes[0].cuda(), codes[1].cuda()
    q = torch.randn(len(ctx), G * hkv, d, generator=g).to(dtype).cuda()
    ks, vs = 0.03, 0.011
    for pt in (0, 16, 64, 512):
        out = torch.empty_like(q)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        ws = pa.decode_workspace(len(ctx), G * hkv, hkv, d, max(ctx), pt)
        pa.pa_paged_decode_fp8(out, q, kc, vc, tables, cl, max(ctx), 0.125, ks, vs, pt, ws, err)
        torch.cuda.synchronize()
        assert err.item() == 0, err.item()
        ref = F.paged_decode_fp8(tensor_bits(q), kc.cpu().numpy(), vc.cpu().numpy(), tab,
                                 np.asarray(ctx), 0.125, ks, vs, name)
        assert_close(out_to_f64(out, name), ref,
                     f"fp8 {os.environ.get('PA_DECODE_PATH')} {os.environ.get('PA_DECODE_SPLIT')} "
                     f"G{G} d{d} {name} pt{pt}")


if __name__ == "__main__":
    main()
