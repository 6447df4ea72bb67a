"""Golden fixtures: small text files, each citing the page or definition it comes from."""
import pathlib

GOLDEN_DIR = pathlib.Path(__file__).resolve().parent


def load_kv(name: str) -> dict:
    """Parse ``key = value`` lines (``#`` starts a comment)."""
    out = {}
    for line in (GOLDEN_DIR / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, val = (s.strip() for s in line.split("=", 1))
        out[key] = float(val)
    return out


def load_rows(name: str) -> list:
    """Whitespace-separated rows, comments stripped."""
    rows = []
    for line in (GOLDEN_DIR / name).read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if line:
            rows.append(line.split())
    return rows
