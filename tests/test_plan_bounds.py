"""Host-side plan of the persistent pass 1 (no GPU needed): the partial-state
slots a (batch, head group) row can touch are counted by brute force over the
balanced CTA ranges, and the library's exported workspace size must hold them for
every CTA count the device can use (its SM count up to the 160-CTA cap), so the
kernel can never write past its partials region.

Pass 1 splits a flat list of T = B * ceil(H / 4) * ceil(N / 64) items (row =
batch x group of 4 heads, 64 tokens per item) over P CTAs, CTA c owning items
[c T / P, (c + 1) T / P); a row's partial slots are the CTAs that own any of its
items.  P is the device's CTA count, reduced so that every CTA has at least 4
items."""
import pytest

import relu_linear_attention_attn_b200 as sla

STAGE_TOK, GROUP, MIN_ITEMS, STATE_BYTES = 64, 4, 4, 32 * 33 * 4


def _slots_needed(B, N, H, P_dev):
    R = -(-N // STAGE_TOK)
    G = -(-H // GROUP)
    T = B * G * R
    P = min(-(-T // MIN_ITEMS), P_dev)
    owner = [0] * T
    for c in range(P):                      # the balanced ranges, enumerated
        for i in range(c * T // P, (c + 1) * T // P):
            owner[i] = c
    return max(len(set(owner[r * R:(r + 1) * R])) for r in range(B * G))


@pytest.mark.parametrize("B,N,H", [(1, 64, 4), (1, 1, 70), (1, 1024, 70), (2, 333, 70),
                                   (8, 4096, 70), (2, 16384, 70), (3, 1000, 5), (1, 65, 1),
                                   (4, 200, 130), (1, 16384, 2), (16, 64, 70), (5, 777, 9)])
def test_workspace_holds_every_row_slot(B, N, H):
    lib = sla.load()
    C = 32 * H
    ws = int(lib.sana_linattn_workspace_bytes(B, N, C, H, 0))
    for P_dev in (132, 148, 160):
        need = B * H * _slots_needed(B, N, H, P_dev) * STATE_BYTES
        assert ws >= need, (B, N, H, P_dev, ws, need)
