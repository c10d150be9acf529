"""Index arithmetic of the ternary kernel that decodes into tensor memory
(ternary_gemm_tc.cu, ternary_gemm_tmem_kernel), re-derived on the host for a
sweep of shapes and cluster splits: every word a producer decodes lies in the
window its group stages, the window fits the 4-byte units copied per row, the
decoder's word phase is one of the five it is specialised for, and the
activation columns split over a cluster in whole units of 4.  No GPU."""
import pytest

K_STAGE = 256      # trits per stage
GROUP = 5          # stages per word group
UNITS = 65         # 4-byte units staged per row and group
SLACK = 16         # bytes allocated past the word buffers
N_ACT = 64         # activation rows (UMMA N)


def words10(k):
    return (k + 9) // 10


def stage_split(kt, ks, rank):
    total = (10 * kt + K_STAGE - 1) // K_STAGE
    share = (total + ks - 1) // ks
    sb = min(rank * share, total)
    se = min(sb + share, total)
    return sb, se


@pytest.mark.parametrize("k", [8, 64, 160, 640, 1288, 1600, 2400, 4096, 4104, 12800, 590496])
@pytest.mark.parametrize("ks", [1, 2, 3, 4])
def test_group_windows_cover_every_decoded_word(k, ks):
    kt = words10(k)
    for rank in range(ks):
        sb, se = stage_split(kt, ks, rank)
        nst = se - sb
        for g in range((nst + GROUP - 1) // GROUP):
            w0 = (K_STAGE * (sb + GROUP * g)) // 10
            for u in range(GROUP):
                jj = GROUP * g + u
                if jj >= nst:
                    break
                for qk in range(4):
                    t0 = K_STAGE * (sb + jj) + 64 * qk
                    jw = t0 // 10
                    phase = t0 - 10 * jw
                    assert phase in (0, 2, 4, 6, 8)
                    rel = jw - w0
                    last = (phase // 2 + 31) // 5  # word of the thread's last pair
                    assert 0 <= rel and rel + last <= 128, (k, ks, rank, g, u, qk)
                    # the staged window: 129 words from a 0- or 2-byte offset in 65 units
                    for off in (0, 2):
                        assert off + 2 * (rel + last) + 2 <= 4 * UNITS
                        # the decoder loads 8 words whatever the phase: in bounds with the slack
                        assert off + 2 * (rel + 7) + 2 <= 4 * UNITS + SLACK


@pytest.mark.parametrize("ks", [1, 2, 3, 4])
def test_cluster_column_blocks(ks):
    units = N_ACT // 4
    begin = [4 * ((units * q) // ks) for q in range(ks + 1)]
    assert begin[0] == 0 and begin[-1] == N_ACT
    widths = [begin[q + 1] - begin[q] for q in range(ks)]
    assert all(w % 4 == 0 and w > 0 for w in widths)
    assert max(widths) <= 4 * ((units + ks - 1) // ks)  # the receive row's width
    # every column has exactly one owner, found the way the kernel finds it
    for col in range(0, N_ACT, 4):
        q = sum(1 for t in range(1, ks) if col >= begin[t])
        assert begin[q] <= col < begin[q + 1]
