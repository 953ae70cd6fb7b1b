"""CPU fp64 oracle of the Samba block: test infrastructure, never on the product path."""
