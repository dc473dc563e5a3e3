"""Per-kernel summary (launches, total device time, share) of an ncu --csv launch list
taken with `--metrics gpu__time_duration.sum`."""
import collections
import csv
import sys

SCALE = {"ns": 1e-6, "nsecond": 1e-6, "us": 1e-3, "usecond": 1e-3, "ms": 1.0, "msecond": 1.0, "s": 1e3,
         "second": 1e3}


def summarize(path):
    rows = list(csv.reader(open(path)))
    hi = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    hdr, data = rows[hi], rows[hi + 1:]
    ki, mi, vi, ui = (hdr.index(c) for c in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    tot, cnt = collections.defaultdict(float), collections.Counter()
    for r in data:
        if len(r) <= vi or r[mi] != "gpu__time_duration.sum":
            continue
        name = r[ki].split("(")[0].split("<")[0].strip()
        tot[name] += float(r[vi].replace(",", "")) * SCALE[r[ui]]
        cnt[name] += 1
    return tot, cnt


if __name__ == "__main__":
    tot, cnt = summarize(sys.argv[1])
    T = sum(tot.values())
    print(f"{'kernel':58s} {'launches':>8s} {'total ms':>12s} {'share':>7s}")
    for n, t in sorted(tot.items(), key=lambda x: -x[1]):
        print(f"{n[:58]:58s} {cnt[n]:8d} {t:12.3f} {100 * t / T:6.2f}%")
    print(f"{'all kernels':58s} {sum(cnt.values()):8d} {T:12.3f}")
