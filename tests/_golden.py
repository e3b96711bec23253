"""Reader for the hand-derived golden fixtures under tests/golden/."""


def read_golden(path):
    """Rows of (exact decimal value, hexadecimal code); '#' lines are comments."""
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = line.split()
            rows.append((float(parts[0]), int(parts[1], 16)))
    return rows
